// attend.cu -- CSA sparse attention and HCA dense attention (split-K).
//
// DeepSeek-V4 summary (b-lab.team), "Core Methodological Innovations" 1:
// CSA attends the top-k selected compressed KV blocks, HCA attends every
// remaining (heavily compressed) entry densely, and both add a sliding
// window of local raw KV entries.  Readings taken: K = V = the 128-d latent
// row; softmax over the union of the selected compressed rows and the
// window rows (no de-duplication); scale * q . x logits.
//
// One query's H heads share every row, so the heads form the M side of the
// tensor-core tiles (16 heads per warp, mma.m16n8k16): S = Q K^T over
// 64-row blocks gathered into shared memory with cp.async (the next block is
// in flight while this one computes), an online softmax in registers, then
// O += P V with P re-packed from the S accumulators.  The attended row list
// of a query is cut into fixed splits (64 rows for CSA, 512 for HCA; never a
// function of the batch, so results are batch invariant); each CTA writes
// its split's (max, sum, unnormalised output) and a combine kernel merges
// the splits in order.
#include "common.cuh"

namespace csa {

constexpr int kCsaRowsPerSplit = 64;    // CSA: k + W rows per query, latency-bound
constexpr int kHcaRowsPerSplit = 256;   // HCA: thousands of rows per query
constexpr int kRowBlock = 64;
constexpr int kRowStride = 136;  // bf16 per smem row (272 B: conflict-free ldmatrix)

struct AttnArgs {
    const bf16* q;
    const int* q_seq;
    const int* q_pos;
    const bf16* comp;
    int64_t comp_stride;
    const bf16* raw;
    int64_t raw_stride;
    int m;
    const int* idx;  // CSA; nullptr for HCA
    int k;
    int max_blocks;  // HCA
    int W;
    float scale_log2;  // scale * log2(e)
    int rows_per_split;
    int nsplit;
    float* part_o;    // [T][nsplit][H][128]
    float* part_ml;   // [T][nsplit][H][2]
    unsigned* status;
};

// Row pointer of list position pos for query (b, p): nullptr = masked.
__device__ __forceinline__ const bf16* row_ptr(const AttnArgs& a, int t, int b, int p, int V, int nsel, int pos) {
    if (pos < nsel) {
        int j;
        if (a.idx) {
            j = a.idx[(int64_t)t * a.k + pos];
            if (j < 0) return nullptr;
            if (j >= V) {
                flag_status(a.status, kDevBadIndex);
                return nullptr;
            }
        } else {
            j = pos;
        }
        return a.comp + (int64_t)b * a.comp_stride + (int64_t)j * 128;
    }
    const int s = p - a.W + 1 + (pos - nsel);
    if (pos - nsel >= a.W || s < 0) return nullptr;
    return a.raw + (int64_t)b * a.raw_stride + (int64_t)s * 128;
}

template <int NW>
__global__ void __launch_bounds__(NW * 32) attend_kernel(AttnArgs a) {
    constexpr int H = NW * 16;
    __shared__ __align__(16) bf16 rows_sh[2][kRowBlock * kRowStride];
    __shared__ int valid_sh[2][kRowBlock];

    const int t = blockIdx.y, sp = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    griddep_wait();
    const int b = a.q_seq[t], p = a.q_pos[t];
    const int V = a.idx ? (p + 1) / a.m : min((p + 1) / a.m, a.max_blocks);
    const int nsel = a.idx ? a.k : V;
    const int total = nsel + a.W;
    const int pos0 = sp * a.rows_per_split;
    const int npos = max(0, min(a.rows_per_split, total - pos0));
    const int nblk = (npos + kRowBlock - 1) / kRowBlock;

    // issue the gather of row block `blk` into buffer `buf`
    auto gather = [&](int blk, int buf) {
        for (int i = threadIdx.x; i < kRowBlock * 16; i += NW * 32) {
            const int r = i >> 4, c = i & 15;
            const int pos = pos0 + blk * kRowBlock + r;
            const bf16* src = nullptr;
            if (blk * kRowBlock + r < npos) src = row_ptr(a, t, b, p, V, nsel, pos);
            cp_async16(&rows_sh[buf][r * kRowStride + c * 8], src ? (const void*)(src + c * 8) : (const void*)a.raw,
                       src ? 16 : 0);
            if (c == 0) valid_sh[buf][r] = src != nullptr;
        }
        cp_async_commit();
    };

    if (nblk > 0) gather(0, 0);

    // Q fragments for this warp's 16 heads: 8 k-steps of 16 dims.
    uint32_t qa[8][4];
    {
        const bf16* qh = a.q + ((int64_t)t * H + warp * 16) * 128;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int c0 = ks * 16 + 2 * tq;
            qa[ks][0] = *reinterpret_cast<const uint32_t*>(qh + (int64_t)g * 128 + c0);
            qa[ks][1] = *reinterpret_cast<const uint32_t*>(qh + (int64_t)(g + 8) * 128 + c0);
            qa[ks][2] = *reinterpret_cast<const uint32_t*>(qh + (int64_t)g * 128 + c0 + 8);
            qa[ks][3] = *reinterpret_cast<const uint32_t*>(qh + (int64_t)(g + 8) * 128 + c0 + 8);
        }
    }

    float o[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

    for (int blk = 0; blk < nblk; ++blk) {
        const int buf = blk & 1;
        if (blk + 1 < nblk) {
            gather(blk + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const bf16* rs = rows_sh[buf];

        // S = Q K^T : 16 heads x 64 rows per warp
        float s[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
                // two k-steps (2kp, 2kp+1) of n-tile j: matrices (rows 8j.., dims 32kp + {0,8,16,24})
                uint32_t bb[4];
                const int mi = lane >> 3, ri = lane & 7;
                ldmatrix_x4(bb, rs + (8 * j + ri) * kRowStride + 32 * kp + 8 * mi);
                mma_bf16_16816(s[j], qa[2 * kp], bb[0], bb[1]);
                mma_bf16_16816(s[j], qa[2 * kp + 1], bb[2], bb[3]);
            }
        }
        // mask + online softmax (log2 domain)
        float bmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = 8 * j + 2 * tq + (e & 1);
                float v = valid_sh[buf][r] ? s[j][e] * a.scale_log2 : -INFINITY;
                s[j][e] = v;
                bmax[e >> 1] = fmaxf(bmax[e >> 1], v);
            }
        }
        float corr[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            bmax[h2] = fmaxf(bmax[h2], __shfl_xor_sync(0xffffffffu, bmax[h2], 1));
            bmax[h2] = fmaxf(bmax[h2], __shfl_xor_sync(0xffffffffu, bmax[h2], 2));
            const float mnew = fmaxf(mrow[h2], bmax[h2]);
            corr[h2] = mnew == -INFINITY ? 1.f : exp2f(mrow[h2] - mnew);
            mrow[h2] = mnew;
        }
        float bsum[2] = {0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float mm = mrow[e >> 1];
                const float pv = mm == -INFINITY ? 0.f : exp2f(s[j][e] - mm);
                s[j][e] = pv;
                bsum[e >> 1] += pv;
            }
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            bsum[h2] += __shfl_xor_sync(0xffffffffu, bsum[h2], 1);
            bsum[h2] += __shfl_xor_sync(0xffffffffu, bsum[h2], 2);
            lrow[h2] = lrow[h2] * corr[h2] + bsum[h2];
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            o[j][0] *= corr[0];
            o[j][1] *= corr[0];
            o[j][2] *= corr[1];
            o[j][3] *= corr[1];
        }
        // O += P V
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t pa[4];
            pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
            pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
            pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int jp = 0; jp < 8; ++jp) {
                // V rows 16kk.., dims 16jp..: matrices (k 0-7,n 0-7),(k 8-15,n 0-7),(k 0-7,n 8-15),(k 8-15,n 8-15)
                uint32_t bb[4];
                const int mi = lane >> 3, ri = lane & 7;
                const int row = 16 * kk + (mi & 1) * 8 + ri;
                const int col = 16 * jp + (mi >> 1) * 8;
                ldmatrix_x4_trans(bb, rs + row * kRowStride + col);
                mma_bf16_16816(o[2 * jp], pa, bb[0], bb[1]);
                mma_bf16_16816(o[2 * jp + 1], pa, bb[2], bb[3]);
            }
        }
        __syncthreads();  // buffer `buf` is refilled two blocks later
    }

    // split partials
    const int h0 = warp * 16 + g;
    float* po = a.part_o + (((int64_t)t * a.nsplit + sp) * H) * 128;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int c = 8 * j + 2 * tq;
        *reinterpret_cast<float2*>(po + (int64_t)h0 * 128 + c) = make_float2(o[j][0], o[j][1]);
        *reinterpret_cast<float2*>(po + (int64_t)(h0 + 8) * 128 + c) = make_float2(o[j][2], o[j][3]);
    }
    if (tq == 0) {
        float* pm = a.part_ml + (((int64_t)t * a.nsplit + sp) * H) * 2;
        pm[h0 * 2] = mrow[0];
        pm[h0 * 2 + 1] = lrow[0];
        pm[(h0 + 8) * 2] = mrow[1];
        pm[(h0 + 8) * 2 + 1] = lrow[1];
    }
    griddep_trigger();
}

// Merge of the split partials of one (query, head) per warp: lane i holds
// split i's (max, sum) -- 32 splits per pass, passes merged in order -- and
// every lane owns 4 output channels, issuing all its splits' partial-output
// loads before summing them in split order.  grid (H / 4, T), 128 threads.
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                                                      int nsplit, int H, bf16* __restrict__ out,
                                                      float* __restrict__ lse) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x * 4 + warp, t = blockIdx.y;
    griddep_wait();
    if (h >= H) return;
    // pass 1: the global max
    float M = -INFINITY;
    for (int base = 0; base < nsplit; base += 32) {
        const int i = base + lane;
        const float mi = i < nsplit ? part_ml[(((int64_t)t * nsplit + i) * H + h) * 2] : -INFINITY;
        M = fmaxf(M, mi);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    // pass 2: factors, sum and output, 32 splits at a time in split order
    float L = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int base = 0; base < nsplit; base += 32) {
        const int i = base + lane;
        float f = 0.f, li = 0.f;
        if (i < nsplit) {
            const int64_t o = (((int64_t)t * nsplit + i) * H + h) * 2;
            const float mi = part_ml[o];
            li = part_ml[o + 1];
            f = (M == -INFINITY || mi == -INFINITY) ? 0.f : exp2f(mi - M);
        }
        const int cnt = min(32, nsplit - base);
        float4 ov[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < cnt)
                ov[j] = *reinterpret_cast<const float4*>(part_o + (((int64_t)t * nsplit + base + j) * H + h) * 128 +
                                                         lane * 4);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if (j < cnt) {
                const float fj = __shfl_sync(0xffffffffu, f, j);
                const float lj = __shfl_sync(0xffffffffu, li, j);
                L = fmaf(lj, fj, L);
                O.x = fmaf(ov[j].x, fj, O.x);
                O.y = fmaf(ov[j].y, fj, O.y);
                O.z = fmaf(ov[j].z, fj, O.z);
                O.w = fmaf(ov[j].w, fj, O.w);
            }
        }
    }
    bf16* op = out + ((int64_t)t * H + h) * 128 + lane * 4;
    const float r0 = L > 0.f ? O.x / L : 0.f, r1 = L > 0.f ? O.y / L : 0.f;
    const float r2 = L > 0.f ? O.z / L : 0.f, r3 = L > 0.f ? O.w / L : 0.f;
    *reinterpret_cast<uint2*>(op) = make_uint2(pack_bf16(r0, r1), pack_bf16(r2, r3));
    if (lse && lane == 0) lse[(int64_t)t * H + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    griddep_trigger();
}

int attend_rows_per_split(bool dense) { return dense ? kHcaRowsPerSplit : kCsaRowsPerSplit; }
int attend_nsplit(int max_rows, bool dense) {
    const int r = attend_rows_per_split(dense);
    return max_rows <= 0 ? 1 : (max_rows + r - 1) / r;
}

cudaError_t launch_attend(const void* q, const int* q_seq, const int* q_pos, int T, int H, const void* comp,
                          int64_t comp_stride, const void* raw, int64_t raw_stride, int m, const int* idx, int k,
                          int max_blocks, int W, float scale, void* out, float* lse, float* part_o,
                          float* part_ml, unsigned* status, bool use_partials, cudaStream_t stream,
                          int* launches) {
    (void)use_partials;   // every split writes partials that combine_kernel merges
    AttnArgs a;
    a.q = reinterpret_cast<const bf16*>(q);
    a.q_seq = q_seq;
    a.q_pos = q_pos;
    a.comp = reinterpret_cast<const bf16*>(comp);
    a.comp_stride = comp_stride;
    a.raw = reinterpret_cast<const bf16*>(raw);
    a.raw_stride = raw_stride;
    a.m = m;
    a.idx = idx;
    a.k = k;
    a.max_blocks = max_blocks;
    a.W = W;
    a.scale_log2 = scale * 1.4426950408889634f;
    const int max_rows = (idx ? k : max_blocks) + W;
    a.rows_per_split = attend_rows_per_split(idx == nullptr);
    a.nsplit = attend_nsplit(max_rows, idx == nullptr);
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.status = status;
    dim3 grid(a.nsplit, T);
    cudaError_t e = cudaSuccess;
    switch (H) {
        case 16: e = launch_pdl(attend_kernel<1>, grid, dim3(32), 0, stream, a); break;
        case 32: e = launch_pdl(attend_kernel<2>, grid, dim3(64), 0, stream, a); break;
        case 48: e = launch_pdl(attend_kernel<3>, grid, dim3(96), 0, stream, a); break;
        case 64: e = launch_pdl(attend_kernel<4>, grid, dim3(128), 0, stream, a); break;
        case 80: e = launch_pdl(attend_kernel<5>, grid, dim3(160), 0, stream, a); break;
        case 96: e = launch_pdl(attend_kernel<6>, grid, dim3(192), 0, stream, a); break;
        case 112: e = launch_pdl(attend_kernel<7>, grid, dim3(224), 0, stream, a); break;
        case 128: e = launch_pdl(attend_kernel<8>, grid, dim3(256), 0, stream, a); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    e = launch_pdl(combine_kernel, dim3((H + 3) / 4, T), dim3(128), 0, stream, (const float*)part_o,
                   (const float*)part_ml, a.nsplit, H, reinterpret_cast<bf16*>(out), lse);
    *launches += 2;
    return e;
}

}  // namespace csa
