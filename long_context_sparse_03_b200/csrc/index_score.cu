// index_score.cu -- lightning-indexer scoring and exact per-query top-k.
//
// DeepSeek-V4 summary (b-lab.team), "Core Methodological Innovations" 1,
// CSA bullet: the "Lightning Indexer" computes scores from low-rank
// projections of h_t and selects the top-k most relevant compressed blocks.
// Readings taken: S_j = sum_h w_h max(0, q_h . k_j) (times the row scale for
// E4M3 keys); block j visible iff j < (p+1)/m; order = score desc, index asc.
//
// Decode is an HBM stream over the compressed indexer keys (64 values per
// block).  Per key it costs Hi*64 multiply-adds in fp32-grade precision,
// which at HBM rate is beyond the CUDA-core fp32 rate, so the dot products
// run on the tensor cores: a warp takes 16 keys as the A operand of
// mma.m16n8k16 (loaded straight from global memory into registers with
// 128-bit coalesced loads) and the query heads as the B operand (n = 8 heads
// per MMA), split into hi + lo halves so the product keeps ~16 significant
// bits of q.  The K dimension (the 64 key channels) is permuted so that each
// lane's fragment is two contiguous 16-byte pieces of a key row; the query
// fragments use the same permutation, so every dot product is unchanged.
//
// Each CTA keeps its chunk's scores on chip as (score, index) keys, selects
// its exact local top-k with a shared-memory radix select and writes only
// those candidates; merge kernels reduce the candidates to the final sorted
// top-k.  The selection is exact under the total order, so the result does
// not depend on how the blocks were chunked (batch invariant).
#include "common.cuh"

namespace csa {

constexpr int kScoreThreads = 256;
constexpr int kMergeThreads = 512;
constexpr int kMergeMax = 16384;  // candidates held by one merge CTA

// ---------------------------------------------------------------- select
// Exact threshold of the kk largest among the distinct nonzero uint64
// values v[0..n) (zero = empty slot).  Returns thr with exactly
// min(kk, #nonzero) values >= thr among the nonzero ones (thr = 1 when all
// are taken).  Every thread of the block must call it.
__device__ uint64_t block_select(const uint64_t* v, int n, int kk, unsigned* hist, int* misc) {
    const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31;
    // count nonzero
    if (tid == 0) misc[2] = 0;
    __syncthreads();
    int cnt = 0;
    for (int i = tid; i < n; i += nth) cnt += v[i] != 0ull;
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if (lane == 0) atomicAdd(&misc[2], cnt);
    __syncthreads();
    const int nz = misc[2];
    if (nz <= kk) return 1ull;

    uint64_t prefix = 0, mask = 0;
    int need = kk;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += nth) hist[i] = 0;
        __syncthreads();
        for (int base = 0; base < n; base += nth) {
            const int i = base + tid;
            uint64_t x = i < n ? v[i] : 0ull;
            const bool match = x != 0ull && (x & mask) == prefix;
            const unsigned dig = (unsigned)(x >> shift) & 255u;
            const unsigned peers = __match_any_sync(0xffffffffu, match ? dig : 0xFFFFFFFFu);
            if (match && lane == __ffs(peers) - 1) atomicAdd(&hist[dig], (unsigned)__popc(peers));
        }
        __syncthreads();
        if (tid < 32) {
            // lane L owns bins 255-8L .. 248-8L (highest first)
            unsigned c[8], s = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                c[e] = hist[255 - 8 * lane - e];
                s += c[e];
            }
            unsigned incl = s;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            const unsigned excl = incl - s;
            if (excl < (unsigned)need && (unsigned)need <= incl) {
                unsigned run = excl;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (run + c[e] >= (unsigned)need) {
                        misc[0] = 255 - 8 * lane - e;
                        misc[1] = (int)run;
                        break;
                    }
                    run += c[e];
                }
            }
        }
        __syncthreads();
        const unsigned d = (unsigned)misc[0];
        const int above = misc[1];
        const unsigned bin = hist[d];
        prefix |= (uint64_t)d << shift;
        mask |= 0xFFull << shift;
        need -= above;
        __syncthreads();  // misc / hist reused next pass
        if ((int)bin == need) break;
    }
    return prefix;
}

// ---------------------------------------------------------------- scoring
// Per-thread query fragments for NT groups of 8 heads.
template <int NT>
struct QFrag {
    uint32_t hi[NT][4][2];
    uint32_t lo[NT][4][2];
    float w[NT][2];
};

// Physical key channel of (k-step s, lane quarter tq, element e) for bf16
// keys: lane tq holds 16-byte chunks tq and tq+4 of the 128-byte row.
__device__ __forceinline__ int phys_bf16(int s, int tq, int e) { return (s >> 1) * 32 + tq * 8 + (s & 1) * 4 + e; }
// ... and for E4M3 keys: lane tq holds 16-byte chunk tq of the 64-byte row.
__device__ __forceinline__ int phys_e4m3(int s, int tq, int e) { return tq * 16 + s * 4 + e; }

template <int FMT, int NT>
__device__ void load_qfrag(QFrag<NT>& f, const float* q_sh, const float* w_sh, const int* e_sh, int Hi) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int hh = nt * 8 + g;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                float x[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int e = rr * 2 + u;
                    const int c = FMT == 0 ? phys_bf16(s, tq, e) : phys_e4m3(s, tq, e);
                    x[u] = hh < Hi ? q_sh[hh * 64 + c] : 0.f;
                }
                if (FMT == 0) {
                    const float h0 = __bfloat162float(__float2bfloat16_rn(x[0]));
                    const float h1 = __bfloat162float(__float2bfloat16_rn(x[1]));
                    f.hi[nt][s][rr] = pack_bf16(h0, h1);
                    f.lo[nt][s][rr] = pack_bf16(x[0] - h0, x[1] - h1);
                } else {
                    const int ex = hh < Hi ? e_sh[hh] : 0;
                    const float y0 = ldexpf(x[0], ex), y1 = ldexpf(x[1], ex);
                    const float h0 = __half2float(__float2half_rn(y0));
                    const float h1 = __half2float(__float2half_rn(y1));
                    f.hi[nt][s][rr] = pack_f16(h0, h1);
                    f.lo[nt][s][rr] = pack_f16(y0 - h0, y1 - h1);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int hc = nt * 8 + 2 * tq + u;  // head of accumulator column 2tq+u
            float wv = hc < Hi ? w_sh[hc] : 0.f;
            if (FMT == 1 && hc < Hi) wv = ldexpf(wv, -e_sh[hc]);
            f.w[nt][u] = wv;
        }
    }
}

// Raw key bytes of one 16-key tile for this lane.
struct KeyTile {
    uint4 a0, a1, b0, b1;  // bf16: rows g, g+8, chunks tq / tq+4; E4M3: a0, a1 only
    float s0, s1;          // E4M3 row scales
};

template <int FMT>
__device__ __forceinline__ void load_tile(KeyTile& kt, const uint8_t* kbase, const float* sbase, int r0, int j1) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int ra = r0 + g, rb = r0 + g + 8;
    const uint4 z = make_uint4(0, 0, 0, 0);
    if (FMT == 0) {
        const uint8_t* pa = kbase + (int64_t)ra * 128 + tq * 16;
        const uint8_t* pb = kbase + (int64_t)rb * 128 + tq * 16;
        kt.a0 = ra < j1 ? ldg_stream(pa) : z;
        kt.b0 = ra < j1 ? ldg_stream(pa + 64) : z;
        kt.a1 = rb < j1 ? ldg_stream(pb) : z;
        kt.b1 = rb < j1 ? ldg_stream(pb + 64) : z;
    } else {
        kt.a0 = ra < j1 ? ldg_stream(kbase + (int64_t)ra * 64 + tq * 16) : z;
        kt.a1 = rb < j1 ? ldg_stream(kbase + (int64_t)rb * 64 + tq * 16) : z;
        kt.s0 = ra < j1 ? __ldg(sbase + ra) : 0.f;
        kt.s1 = rb < j1 ? __ldg(sbase + rb) : 0.f;
    }
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xFFFFu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Scores of the lane's two rows (g, g+8) of one tile (valid in every lane
// of the quad after the reduction).
template <int FMT, int NT>
__device__ __forceinline__ void score_tile(const KeyTile& kt, const QFrag<NT>& f, float& s0, float& s1) {
    float c[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t a[4];
        if (FMT == 0) {
            const uint4& A = (s < 2) ? kt.a0 : kt.b0;
            const uint4& Bq = (s < 2) ? kt.a1 : kt.b1;
            const bool hiw = s & 1;
            a[0] = hiw ? A.z : A.x;
            a[2] = hiw ? A.w : A.y;
            a[1] = hiw ? Bq.z : Bq.x;
            a[3] = hiw ? Bq.w : Bq.y;
        } else {
            const uint32_t wa = s == 0 ? kt.a0.x : s == 1 ? kt.a0.y : s == 2 ? kt.a0.z : kt.a0.w;
            const uint32_t wb = s == 0 ? kt.a1.x : s == 1 ? kt.a1.y : s == 2 ? kt.a1.z : kt.a1.w;
            a[0] = e4m3x2_to_f16x2(wa);
            a[2] = e4m3x2_to_f16x2(wa >> 16);
            a[1] = e4m3x2_to_f16x2(wb);
            a[3] = e4m3x2_to_f16x2(wb >> 16);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            if (FMT == 0) {
                mma_bf16_16816(c[nt], a, f.hi[nt][s][0], f.hi[nt][s][1]);
                mma_bf16_16816(c[nt], a, f.lo[nt][s][0], f.lo[nt][s][1]);
            } else {
                mma_f16_16816(c[nt], a, f.hi[nt][s][0], f.hi[nt][s][1]);
                mma_f16_16816(c[nt], a, f.lo[nt][s][0], f.lo[nt][s][1]);
            }
        }
    }
    float p0 = 0.f, p1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        p0 = fmaf(f.w[nt][0], fmaxf(c[nt][0], 0.f), p0);
        p0 = fmaf(f.w[nt][1], fmaxf(c[nt][1], 0.f), p0);
        p1 = fmaf(f.w[nt][0], fmaxf(c[nt][2], 0.f), p1);
        p1 = fmaf(f.w[nt][1], fmaxf(c[nt][3], 0.f), p1);
    }
    p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
    p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
    p0 += __shfl_xor_sync(0xffffffffu, p0, 2);
    p1 += __shfl_xor_sync(0xffffffffu, p1, 2);
    if (FMT == 1) {
        p0 *= kt.s0;
        p1 *= kt.s1;
    }
    s0 = p0;
    s1 = p1;
}

// grid (nchunks, T), 256 threads.  MODE 0: write exact local top-kc
// candidates of the chunk to cand[t][chunk][kc].  MODE 1: write the raw
// scores to scores[t][max_blocks] (NaN past V(t)).
template <int FMT, int NT, int MODE>
__global__ void __launch_bounds__(kScoreThreads, 2) index_score_kernel(
    const float* __restrict__ q, const float* __restrict__ w, const int* __restrict__ q_seq,
    const int* __restrict__ q_pos, int Hi, const uint8_t* __restrict__ kidx,
    const float* __restrict__ kscale, int64_t kstride_bytes, int64_t sstride, int m, int max_blocks,
    int chunk, int kc, uint64_t* __restrict__ cand, float* __restrict__ scores) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t* cand_sh = reinterpret_cast<uint64_t*>(smem_raw);             // [chunk]
    float* q_sh = reinterpret_cast<float*>(smem_raw + (size_t)chunk * 8);  // [16*64]
    float* w_sh = q_sh + 16 * 64;                                          // [16]
    int* e_sh = reinterpret_cast<int*>(w_sh + 16);                         // [16]
    unsigned* hist = reinterpret_cast<unsigned*>(e_sh + 16);               // [256]
    int* misc = reinterpret_cast<int*>(hist + 256);                        // [4]

    const int t = blockIdx.y, ch = blockIdx.x;
    const int b = q_seq[t];
    const int V = min((q_pos[t] + 1) / m, max_blocks);
    const int j0 = ch * chunk;
    const int j1 = min(j0 + chunk, V);
    const int n = max(0, j1 - j0);

    if (MODE == 1) {
        for (int j = max(j0, V) + threadIdx.x; j < min(j0 + chunk, max_blocks); j += blockDim.x)
            scores[(int64_t)t * max_blocks + j] = __int_as_float(0x7fc00000);
    }
    if (n == 0) {
        if (MODE == 0)
            for (int i = threadIdx.x; i < kc; i += blockDim.x) cand[((int64_t)t * gridDim.x + ch) * kc + i] = 0ull;
        return;
    }

    for (int i = threadIdx.x; i < Hi * 64; i += blockDim.x) q_sh[i] = q[(int64_t)t * Hi * 64 + i];
    if (threadIdx.x < Hi) w_sh[threadIdx.x] = w[(int64_t)t * Hi + threadIdx.x];
    __syncthreads();
    if (FMT == 1 && threadIdx.x < Hi) {
        // power-of-two scale per head so its largest |q| sits in [2^14, 2^15)
        float amax = 0.f;
        for (int c = 0; c < 64; ++c) amax = fmaxf(amax, fabsf(q_sh[threadIdx.x * 64 + c]));
        int ex = 0;
        if (amax > 0.f) {
            int e2;
            frexpf(amax, &e2);
            ex = 15 - e2;
        }
        e_sh[threadIdx.x] = ex;
    }
    __syncthreads();

    QFrag<NT> f;
    load_qfrag<FMT, NT>(f, q_sh, w_sh, e_sh, Hi);

    const uint8_t* kbase = kidx + (int64_t)b * kstride_bytes;
    const float* sbase = FMT == 1 ? kscale + (int64_t)b * sstride : nullptr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int ntiles = (n + 15) >> 4;

    // two tiles per step, the next pair prefetched while this one computes
    KeyTile cur[2], nxt[2];
    int tile = warp;
#pragma unroll
    for (int u = 0; u < 2; ++u)
        if (tile + 8 * u < ntiles) load_tile<FMT>(cur[u], kbase, sbase, j0 + (tile + 8 * u) * 16, j1);
    for (; tile < ntiles; tile += 16) {
#pragma unroll
        for (int u = 0; u < 2; ++u)
            if (tile + 16 + 8 * u < ntiles) load_tile<FMT>(nxt[u], kbase, sbase, j0 + (tile + 16 + 8 * u) * 16, j1);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int tl = tile + 8 * u;
            if (tl < ntiles) {
                float s0, s1;
                score_tile<FMT, NT>(cur[u], f, s0, s1);
                const int ra = j0 + tl * 16 + g, rb = ra + 8;
                if (tq == 0) {
                    if (MODE == 0) {
                        if (ra < j1) cand_sh[ra - j0] = make_cand(s0, ra);
                        if (rb < j1) cand_sh[rb - j0] = make_cand(s1, rb);
                    } else {
                        if (ra < j1) scores[(int64_t)t * max_blocks + ra] = s0;
                        if (rb < j1) scores[(int64_t)t * max_blocks + rb] = s1;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) cur[u] = nxt[u];
    }
    if (MODE == 1) return;
    __syncthreads();

    uint64_t* dst = cand + ((int64_t)t * gridDim.x + ch) * kc;
    if (n <= kc) {
        for (int i = threadIdx.x; i < kc; i += blockDim.x) dst[i] = i < n ? cand_sh[i] : 0ull;
        return;
    }
    const uint64_t thr = block_select(cand_sh, n, kc, hist, misc);
    if (threadIdx.x == 0) misc[3] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const uint64_t x = cand_sh[i];
        if (x >= thr) dst[atomicAdd(&misc[3], 1)] = x;
    }
}

// ---------------------------------------------------------------- merge
// grid (ngroups, T).  CTA takes candidates [g*group, min((g+1)*group, n)) of
// query t.  FINAL: sort the top-k (score desc, index asc) and write
// out_idx / out_score; else write k candidates to out[t][g][k].
template <bool FINAL>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const uint64_t* __restrict__ in, int n, int group,
                                                              int k, uint64_t* __restrict__ out,
                                                              int* __restrict__ out_idx,
                                                              float* __restrict__ out_score) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t* v = reinterpret_cast<uint64_t*>(smem_raw);  // [group]
    unsigned* hist = reinterpret_cast<unsigned*>(v + group);
    int* misc = reinterpret_cast<int*>(hist + 256);
    uint64_t* srt = reinterpret_cast<uint64_t*>(misc + 8);  // [P] (FINAL)

    const int t = blockIdx.y, gi = blockIdx.x;
    const int lo = gi * group, cnt = min(group, n - lo);
    const uint64_t* src = in + (int64_t)t * n + lo;
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) v[i] = src[i];
    __syncthreads();
    const uint64_t thr = block_select(v, cnt, k, hist, misc);

    if (!FINAL) {
        uint64_t* dst = out + ((int64_t)t * gridDim.x + gi) * k;
        if (threadIdx.x == 0) misc[3] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
            const uint64_t x = v[i];
            if (x != 0ull && x >= thr) dst[atomicAdd(&misc[3], 1)] = x;
        }
        __syncthreads();
        for (int i = misc[3] + threadIdx.x; i < k; i += blockDim.x) dst[i] = 0ull;
        return;
    }
    int P = 1;
    while (P < k) P <<= 1;
    for (int i = threadIdx.x; i < P; i += blockDim.x) srt[i] = 0ull;
    if (threadIdx.x == 0) misc[3] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
        const uint64_t x = v[i];
        if (x != 0ull && x >= thr) srt[atomicAdd(&misc[3], 1)] = x;
    }
    __syncthreads();
    // bitonic sort, descending
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < P / 2; i += blockDim.x) {
                const int pos = 2 * i - (i & (stride - 1));
                const int par = pos + stride;
                const bool desc = (pos & size) == 0;
                const uint64_t x = srt[pos], y = srt[par];
                if ((x < y) == desc) {
                    srt[pos] = y;
                    srt[par] = x;
                }
            }
            __syncthreads();
        }
    }
    const int nsel = misc[3];
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const uint64_t x = srt[i];
        const bool ok = i < nsel;
        out_idx[(int64_t)t * k + i] = ok ? cand_index(x) : -1;
        if (out_score) out_score[(int64_t)t * k + i] = ok ? cand_score(x) : __int_as_float(0x7fc00000);
    }
}

// ---------------------------------------------------------------- host
int score_chunk(int T, int max_blocks) {
    for (int c = 8192; c > 1024; c >>= 1)
        if ((int64_t)T * ((max_blocks + c - 1) / c) >= 512) return c;
    return 1024;
}

struct SelectPlan {
    int chunk, nchunks, kc;
    int64_t n0;              // candidates per query after scoring
    size_t cand_a, cand_b;   // bytes of the two candidate buffers
};

SelectPlan plan_select(int T, int max_blocks, int k) {
    SelectPlan p;
    p.chunk = score_chunk(T, max_blocks);
    p.nchunks = (max_blocks + p.chunk - 1) / p.chunk;
    if (p.nchunks < 1) p.nchunks = 1;
    p.kc = k < p.chunk ? k : p.chunk;
    p.n0 = (int64_t)p.nchunks * p.kc;
    p.cand_a = (size_t)T * (size_t)p.n0 * 8;
    int64_t n = p.n0, maxb = 0;
    while (n > kMergeMax) {
        const int64_t ng = (n + kMergeMax - 1) / kMergeMax;
        n = ng * k;
        if (n > maxb) maxb = n;
    }
    p.cand_b = (size_t)T * (size_t)maxb * 8;
    return p;
}

static size_t score_smem(int chunk) { return (size_t)chunk * 8 + 16 * 64 * 4 + 16 * 4 + 16 * 4 + 256 * 4 + 16; }

cudaError_t launch_index_score(const float* q, const float* w, const int* q_seq, const int* q_pos, int T, int Hi,
                               const void* kidx, int fmt, const float* kscale, int64_t kstride_elems,
                               int64_t sstride, int m, int max_blocks, int k, uint64_t* cand, float* scores,
                               cudaStream_t stream, int* launches) {
    const SelectPlan p = plan_select(T, max_blocks, k);
    const int chunk = p.chunk;
    dim3 grid(p.nchunks, T);
    const size_t smem = score_smem(chunk);
    const int64_t kbytes = kstride_elems * (fmt == 0 ? 2 : 1);
    const uint8_t* kb = reinterpret_cast<const uint8_t*>(kidx);
    const bool dbg = scores != nullptr;
    const int nt = Hi > 8 ? 2 : 1;
#define CSA_LAUNCH_SCORE(F, N, MD)                                                                      \
    do {                                                                                                \
        auto kern = index_score_kernel<F, N, MD>;                                                       \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        if (e != cudaSuccess) return e;                                                                 \
        kern<<<grid, kScoreThreads, smem, stream>>>(q, w, q_seq, q_pos, Hi, kb, kscale, kbytes, sstride, m, \
                                                    max_blocks, chunk, p.kc, cand, scores);             \
    } while (0)
    if (fmt == 0) {
        if (nt == 1) { if (dbg) CSA_LAUNCH_SCORE(0, 1, 1); else CSA_LAUNCH_SCORE(0, 1, 0); }
        else         { if (dbg) CSA_LAUNCH_SCORE(0, 2, 1); else CSA_LAUNCH_SCORE(0, 2, 0); }
    } else {
        if (nt == 1) { if (dbg) CSA_LAUNCH_SCORE(1, 1, 1); else CSA_LAUNCH_SCORE(1, 1, 0); }
        else         { if (dbg) CSA_LAUNCH_SCORE(1, 2, 1); else CSA_LAUNCH_SCORE(1, 2, 0); }
    }
#undef CSA_LAUNCH_SCORE
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_index_merge(int T, int max_blocks, int k, uint64_t* cand_a, uint64_t* cand_b, int* out_idx,
                               float* out_score, cudaStream_t stream, int* launches) {
    const SelectPlan p = plan_select(T, max_blocks, k);
    int64_t n = p.n0;
    uint64_t* src = cand_a;
    uint64_t* dst = cand_b;
    while (n > kMergeMax) {
        const int ng = (int)((n + kMergeMax - 1) / kMergeMax);
        const size_t smem = (size_t)kMergeMax * 8 + 256 * 4 + 32;
        auto kern = merge_kernel<false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3(ng, T), kMergeThreads, smem, stream>>>(src, (int)n, kMergeMax, k, dst, nullptr, nullptr);
        *launches += 1;
        n = (int64_t)ng * k;
        uint64_t* tmp = src;
        src = dst;
        dst = tmp;
    }
    int P = 1;
    while (P < k) P <<= 1;
    const size_t smem = (size_t)n * 8 + 256 * 4 + 32 + (size_t)P * 8;
    auto kern = merge_kernel<true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(1, T), kMergeThreads, smem, stream>>>(src, (int)n, (int)n, k, nullptr, out_idx, out_score);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace csa
