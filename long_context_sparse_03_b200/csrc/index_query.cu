// index_query.cu -- the lightning indexer's query projection.
//
// DeepSeek-V4 summary (b-lab.team), "Core Methodological Innovations" 1,
// CSA bullet: the indexer scores blocks "using low-rank projections of query
// hidden states h_t".  Reading taken: u = W_dq h (rank r), q_h = W_uq[h] u,
// and the per-head weights w = W_w h; u, q and w stay in fp32.
//
// At decode this is a GEMV over the weights (4-5 MB), so the kernel is
// organised for memory-level parallelism: one warp per weight row, every
// lane issuing its 16-byte weight loads up front, and the (small) input
// vectors of up to 8 queries staged once per CTA in shared memory.  Each
// lane accumulates its share in fp32 FMA order, then a fixed-order warp
// reduction finishes the dot product (deterministic).
#include "common.cuh"

namespace csa {

constexpr int kGemvTT = 8;       // queries per pass
constexpr int kGemvBatch = 16;   // 16-byte weight chunks in flight per lane
constexpr int kGemvRows = 4;     // weight rows (warps) per CTA

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float* x) {
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(b[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}

// Stage X[t0 .. t0+TT)[0..K) into shared memory (its own type) with
// cp.async, so every 16-byte piece is in flight at once; rows past T are
// zero-filled.
template <typename XT>
__device__ __forceinline__ void stage_x(XT* xs, const XT* X, int T, int t0, int K) {
    constexpr int per16 = 16 / sizeof(XT);
    const int n16 = K / per16;
    for (int i = threadIdx.x; i < kGemvTT * n16; i += blockDim.x) {
        const int u = i / n16, c = (i % n16) * per16;
        const bool ok = t0 + u < T;
        cp_async16(xs + (size_t)u * K + c, ok ? (const void*)(X + (int64_t)(t0 + u) * K + c) : (const void*)X,
                   ok ? 16 : 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
}

__device__ __forceinline__ void load8x(const bf16* p, float* x) { bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), x); }
__device__ __forceinline__ void load8x(const float* p, float* x) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Y[t][row] = sum_c W[row][c] X[t][c]: rows of W0 (n0 rows) then W1 (n1 rows),
// written to Y0 (ld0) and Y1 (ld1).  One warp per row, kGemvRows rows per CTA.
template <typename XT>
__global__ void __launch_bounds__(kGemvRows * 32) gemv_kernel(const bf16* __restrict__ W0, int n0, float* __restrict__ Y0,
                                                   int ld0, const bf16* __restrict__ W1, int n1,
                                                   float* __restrict__ Y1, int ld1, int K,
                                                   const XT* __restrict__ X, int T) {
    extern __shared__ __align__(16) uint8_t xs_raw[];
    XT* xs = reinterpret_cast<XT*>(xs_raw);  // [kGemvTT][K]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kGemvRows + warp;
    const bf16* wr = nullptr;
    float* yr = nullptr;
    int ld = 0;
    if (row < n0) {
        wr = W0 + (int64_t)row * K;
        yr = Y0 + row;
        ld = ld0;
    } else if (row < n0 + n1) {
        wr = W1 + (int64_t)(row - n0) * K;
        yr = Y1 + (row - n0);
        ld = ld1;
    }
    const int nchunk = K / 8;
    griddep_wait();
    for (int t0 = 0; t0 < T; t0 += kGemvTT) {
        __syncthreads();
        stage_x<XT>(xs, X, T, t0, K);
        __syncthreads();
        if (!wr) continue;
        float acc[kGemvTT];
#pragma unroll
        for (int u = 0; u < kGemvTT; ++u) acc[u] = 0.f;
        for (int c0 = lane; c0 < nchunk; c0 += 32 * kGemvBatch) {
            uint4 wv[kGemvBatch];
#pragma unroll
            for (int b = 0; b < kGemvBatch; ++b) {
                const int c = c0 + 32 * b;
                wv[b] = c < nchunk ? ldg_stream(wr + (int64_t)c * 8) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int b = 0; b < kGemvBatch; ++b) {
                const int c = c0 + 32 * b;
                if (c < nchunk) {
                    float wf[8];
                    bf16x8_to_f32(wv[b], wf);
#pragma unroll
                    for (int u = 0; u < kGemvTT; ++u) {
                        float xv[8];
                        load8x(xs + (size_t)u * K + c * 8, xv);
                        float s = acc[u];
#pragma unroll
                        for (int e = 0; e < 8; ++e) s = fmaf(wf[e], xv[e], s);
                        acc[u] = s;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kGemvTT; ++u) {
            float v = acc[u];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            if (lane == 0 && t0 + u < T) yr[(int64_t)(t0 + u) * ld] = v;
        }
    }
    griddep_trigger();
}

// ---------------------------------------------------------------- tensor-core GEMV
// Y[t][row] = sum_c W[row][c] X[t][c] for bf16 W and bf16 X (exact bf16
// products, fp32 accumulation) on mma.m16n8k16: a warp takes 16 weight rows
// as the A operand, loaded straight from global memory into registers
// (lane quarter tq holds 16-byte chunks tq and tq+4 of every 64-element
// block of rows g and g+8), and up to 8 queries as B, read from the staged
// copy of X with the same channel permutation.  The CTA's 16 warps split K
// evenly; their 16 x 8 partial tiles are summed in warp order (fixed, so
// deterministic).  Used when K is a multiple of 1024 (64 channels x 16
// warps); other K use the SIMT kernel above.
constexpr int kMmaWarps = 16;

// Stage X[t0 .. t0+8)[0..K) (bf16) into shared memory already laid out as
// B fragments: the 8 bytes lane (g, tq) needs for k-step s of 64-channel
// block b -- channels b*64 + (s>>1)*32 + tq*8 + (s&1)*4 .. +4 of query g --
// sit at 8-byte slot ((b*4 + s)*4 + tq)*8 + g, so a warp's fragment load is
// 256 contiguous bytes (no bank conflicts).  Queries past T read as zero.
__device__ __forceinline__ void stage_x_frag(uint2* xs, const bf16* X, int T, int t0, int K) {
    const int nslot = (K / 4) * kGemvTT;   // 8-byte slots
    for (int i = threadIdx.x; i < nslot; i += blockDim.x) {
        const int g = i & 7, tq = (i >> 3) & 3, s = (i >> 5) & 3, b = i >> 7;
        const int c = b * 64 + (s >> 1) * 32 + tq * 8 + (s & 1) * 4;
        const bool ok = t0 + g < T;
        const uint32_t d = (uint32_t)__cvta_generic_to_shared(xs + i);
        const void* src = ok ? (const void*)(X + (int64_t)(t0 + g) * K + c) : (const void*)X;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(d), "l"(src), "r"(ok ? 8 : 0));
    }
    cp_async_commit();
    cp_async_wait<0>();
}

__global__ void __launch_bounds__(kMmaWarps * 32) gemv_mma_kernel(const bf16* __restrict__ W0, int n0,
                                                                 float* __restrict__ Y0, int ld0,
                                                                 const bf16* __restrict__ W1, int n1,
                                                                 float* __restrict__ Y1, int ld1, int K,
                                                                 const bf16* __restrict__ X, int T) {
    extern __shared__ __align__(16) uint8_t smem_g[];
    uint2* xs = reinterpret_cast<uint2*>(smem_g);                                 // B fragments, 16 * K bytes
    float* part = reinterpret_cast<float*>(smem_g + (size_t)kGemvTT * K * 2);     // [kMmaWarps][16][8]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int row0 = blockIdx.x * 16;
    const int KW = K / kMmaWarps;               // channels per warp (multiple of 64)
    const int c_lo = warp * KW;
    // the two weight rows of this lane (rows past n0 + n1 read as zero)
    auto wrow = [&](int r) -> const bf16* {
        if (r < n0) return W0 + (int64_t)r * K;
        if (r < n0 + n1) return W1 + (int64_t)(r - n0) * K;
        return nullptr;
    };
    const bf16* wa = wrow(row0 + g);
    const bf16* wb = wrow(row0 + g + 8);
    griddep_wait();
    for (int t0 = 0; t0 < T; t0 += kGemvTT) {
        __syncthreads();
        stage_x_frag(xs, X, T, t0, K);
        __syncthreads();
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        for (int cb = c_lo; cb < c_lo + KW; cb += 256) {
            // four 64-channel blocks: 16 loads of 16 bytes in flight per lane
            uint4 a[4][4];
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int bk = 0; bk < 4; ++bk) {
                const int cc = cb + bk * 64;
                const bool in = cc < c_lo + KW;
                a[bk][0] = (in && wa) ? ldg_stream(wa + cc + tq * 8) : z;        // row g, chunk tq
                a[bk][1] = (in && wa) ? ldg_stream(wa + cc + 32 + tq * 8) : z;   // row g, chunk tq+4
                a[bk][2] = (in && wb) ? ldg_stream(wb + cc + tq * 8) : z;        // row g+8, chunk tq
                a[bk][3] = (in && wb) ? ldg_stream(wb + cc + 32 + tq * 8) : z;   // row g+8, chunk tq+4
            }
#pragma unroll
            for (int bk = 0; bk < 4; ++bk) {
                const int cc = cb + bk * 64;
                if (cc >= c_lo + KW) break;
                const uint2* xb = xs + (size_t)(cc / 64) * 128 + tq * 8 + g;
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    // channels of k-step s for lane tq: (s>>1)*32 + tq*8 + (s&1)*4 + {0..3}
                    const uint4& A = (s < 2) ? a[bk][0] : a[bk][1];
                    const uint4& B = (s < 2) ? a[bk][2] : a[bk][3];
                    const bool hiw = s & 1;
                    uint32_t af[4];
                    af[0] = hiw ? A.z : A.x;
                    af[2] = hiw ? A.w : A.y;
                    af[1] = hiw ? B.z : B.x;
                    af[3] = hiw ? B.w : B.y;
                    const uint2 bb = xb[s * 32];
                    mma_bf16_16816(c, af, bb.x, bb.y);
                }
            }
        }
        // c: (row g, queries 2tq, 2tq+1), (row g+8, same queries)
        float* pw = part + warp * 128;
        pw[g * 8 + 2 * tq] = c[0];
        pw[g * 8 + 2 * tq + 1] = c[1];
        pw[(g + 8) * 8 + 2 * tq] = c[2];
        pw[(g + 8) * 8 + 2 * tq + 1] = c[3];
        __syncthreads();
        if (threadIdx.x < 128) {
            const int rr = threadIdx.x >> 3, u = threadIdx.x & 7;
            float acc = 0.f;
            for (int w2 = 0; w2 < kMmaWarps; ++w2) acc += part[w2 * 128 + rr * 8 + u];
            const int r = row0 + rr;
            if (t0 + u < T) {
                if (r < n0) Y0[(int64_t)(t0 + u) * ld0 + r] = acc;
                else if (r < n0 + n1) Y1[(int64_t)(t0 + u) * ld1 + (r - n0)] = acc;
            }
        }
    }
    griddep_trigger();
}

template <typename XT>
static cudaError_t launch_gemv(const bf16* W0, int n0, float* Y0, int ld0, const bf16* W1, int n1, float* Y1, int ld1,
                               int K, const XT* X, int T, cudaStream_t stream) {
    const size_t smem = sizeof(XT) * kGemvTT * (size_t)K;
    auto kern = gemv_kernel<XT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, dim3((n0 + n1 + kGemvRows - 1) / kGemvRows), dim3(kGemvRows * 32), smem, stream, W0, n0,
                      Y0, ld0, W1, n1, Y1, ld1, K, X, T);
}

template <typename AT>
cudaError_t launch_gemm_tn(const AT* A, int M, int K, const bf16* B0, int n0, float* C0, int ldc0, const bf16* B1,
                           int n1, float* C1, int ldc1, cudaStream_t stream);

// Many queries (chunked prefill): the projections are tiled GEMMs.
constexpr int kGemmMinT = 64;

// q_out [T][Hi*64], w_out [T][Hi], u_ws [T][r] (fp32 scratch).
cudaError_t launch_index_query(const void* h, int T, int D, int r, int Hi, const void* W_dq, const void* W_uq,
                               const void* W_w, float* q_out, float* w_out, float* u_ws, cudaStream_t stream,
                               int* launches) {
    const bf16* hb = reinterpret_cast<const bf16*>(h);
    cudaError_t e;
    if (T >= kGemmMinT && D % 32 == 0 && r % 32 == 0) {
        e = launch_gemm_tn<bf16>(hb, T, D, reinterpret_cast<const bf16*>(W_dq), r, u_ws, r,
                                 reinterpret_cast<const bf16*>(W_w), Hi, w_out, Hi, stream);
        if (e != cudaSuccess) return e;
        e = launch_gemm_tn<float>(u_ws, T, r, reinterpret_cast<const bf16*>(W_uq), Hi * 64, q_out, Hi * 64, nullptr, 0,
                                  nullptr, 0, stream);
        *launches += 2;
        return e;
    }
    if (D % (64 * kMmaWarps) == 0) {
        const size_t smem = (size_t)kGemvTT * D * 2 + (size_t)kMmaWarps * 128 * 4;
        e = cudaFuncSetAttribute(gemv_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(gemv_mma_kernel, dim3((r + Hi + 15) / 16), dim3(kMmaWarps * 32), smem, stream,
                       reinterpret_cast<const bf16*>(W_dq), r, u_ws, r, reinterpret_cast<const bf16*>(W_w), Hi,
                       w_out, Hi, D, hb, T);
    } else {
        e = launch_gemv<bf16>(reinterpret_cast<const bf16*>(W_dq), r, u_ws, r, reinterpret_cast<const bf16*>(W_w), Hi,
                              w_out, Hi, D, hb, T, stream);
    }
    if (e != cudaSuccess) return e;
    e = launch_gemv<float>(reinterpret_cast<const bf16*>(W_uq), Hi * 64, q_out, Hi * 64, nullptr, 0, nullptr, 0, r,
                           u_ws, T, stream);
    *launches += 2;
    return e;
}

}  // namespace csa
