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
    kern<<<(n0 + n1 + kGemvRows - 1) / kGemvRows, kGemvRows * 32, smem, stream>>>(W0, n0, Y0, ld0, W1, n1, Y1, ld1,
                                                                                  K, X, T);
    return cudaGetLastError();
}

// q_out [T][Hi*64], w_out [T][Hi], u_ws [T][r] (fp32 scratch).
cudaError_t launch_index_query(const void* h, int T, int D, int r, int Hi, const void* W_dq, const void* W_uq,
                               const void* W_w, float* q_out, float* w_out, float* u_ws, cudaStream_t stream,
                               int* launches) {
    const bf16* hb = reinterpret_cast<const bf16*>(h);
    cudaError_t e = launch_gemv<bf16>(reinterpret_cast<const bf16*>(W_dq), r, u_ws, r,
                                      reinterpret_cast<const bf16*>(W_w), Hi, w_out, Hi, D, hb, T, stream);
    if (e != cudaSuccess) return e;
    e = launch_gemv<float>(reinterpret_cast<const bf16*>(W_uq), Hi * 64, q_out, Hi * 64, nullptr, 0, nullptr, 0, r,
                           u_ws, T, stream);
    *launches += 2;
    return e;
}

}  // namespace csa
