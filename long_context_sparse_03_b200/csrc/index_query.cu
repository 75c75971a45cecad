// index_query.cu -- the lightning indexer's query projection.
//
// DeepSeek-V4 summary (b-lab.team), "Core Methodological Innovations" 1,
// CSA bullet: the indexer scores blocks "using low-rank projections of query
// hidden states h_t".  Reading taken: u = W_dq h (rank r), q_h = W_uq[h] u,
// and the per-head weights w = W_w h; u, q and w stay in fp32.
//
// At decode this is a GEMV over the weights (each weight row is read once
// and dotted with every query's input, which sits in L1/L2): one warp per
// output row, 16-byte loads, fp32 FMA, a fixed-order warp reduction.
#include "common.cuh"

namespace csa {

template <typename XT>
__device__ __forceinline__ void load8(const XT* p, float* x);

template <>
__device__ __forceinline__ void load8<bf16>(const bf16* p, float* x) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(b[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float* x) {
    float4 a = *reinterpret_cast<const float4*>(p);
    float4 b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Y[t][row] = sum_c W[row][c] X[t][c] for rows < nrows, t < T.
template <typename XT, int TT>
__global__ void __launch_bounds__(256) gemv_kernel(const bf16* __restrict__ Wm, int nrows, int K,
                                                   const XT* __restrict__ X, int T,
                                                   float* __restrict__ Y, int ldy) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= nrows) return;
    const bf16* wr = Wm + (int64_t)row * K;
    for (int t0 = 0; t0 < T; t0 += TT) {
        float acc[TT];
#pragma unroll
        for (int u = 0; u < TT; ++u) acc[u] = 0.f;
        for (int c = lane * 8; c < K; c += 256) {
            float wv[8];
            load8<bf16>(wr + c, wv);
#pragma unroll
            for (int u = 0; u < TT; ++u) {
                if (t0 + u < T) {
                    float xv[8];
                    load8<XT>(X + (int64_t)(t0 + u) * K + c, xv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[u] = fmaf(wv[e], xv[e], acc[u]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < TT; ++u) {
            float v = acc[u];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            if (lane == 0 && t0 + u < T) Y[(int64_t)(t0 + u) * ldy + row] = v;
        }
    }
}

// q_out [T][Hi*64], w_out [T][Hi], u_ws [T][r] (fp32 scratch).
cudaError_t launch_index_query(const void* h, int T, int D, int r, int Hi, const void* W_dq,
                               const void* W_uq, const void* W_w, float* q_out, float* w_out,
                               float* u_ws, cudaStream_t stream, int* launches) {
    const bf16* hb = reinterpret_cast<const bf16*>(h);
    gemv_kernel<bf16, 8><<<(r + 7) / 8, 256, 0, stream>>>(reinterpret_cast<const bf16*>(W_dq), r, D, hb,
                                                          T, u_ws, r);
    gemv_kernel<bf16, 8><<<(Hi + 7) / 8, 256, 0, stream>>>(reinterpret_cast<const bf16*>(W_w), Hi, D, hb,
                                                           T, w_out, Hi);
    gemv_kernel<float, 8><<<(Hi * 64 + 7) / 8, 256, 0, stream>>>(reinterpret_cast<const bf16*>(W_uq),
                                                                 Hi * 64, r, u_ws, T, q_out, Hi * 64);
    *launches += 3;
    return cudaGetLastError();
}

}  // namespace csa
