// gemm.cu -- the indexer query projection for many queries (chunked prefill).
//
// DeepSeek-V4 summary (b-lab.team), "Core Methodological Innovations" 1,
// CSA bullet: the indexer works on low-rank projections of the query hidden
// states h_t.  With thousands of queries the projections u = h W_dq^T,
// w = h W_w^T and q = u W_uq^T are dense GEMMs: C[t][o] = sum_c A[t][c] B[o][c]
// with both operands K-major.  A is bf16 (h) or fp32 (u: split into a bf16
// hi + lo pair so the product keeps ~16 significant bits of u), B is bf16;
// products are exact and accumulation is fp32 on mma.m16n8k16.
//
// Tiles of 128 (queries) x 64 (outputs) x 32 (channels), 8 warps each owning
// 32 x 32, operands staged with cp.async into padded shared rows (conflict-
// free ldmatrix) and double-buffered over K.  B rows are drawn from two
// matrices (W_dq then W_w) and the outputs written to two arrays, so u and w
// come from one launch.
#include "common.cuh"

namespace csa {

constexpr int kGBM = 128, kGBN = 64, kGBK = 32;
constexpr int kGPadBf = 40;   // bf16 per shared row of A / B (80 B)
constexpr int kGPadF = 36;    // floats per shared row of fp32 A (144 B)

template <typename AT>
struct GemmSmem;
template <>
struct GemmSmem<bf16> {
    bf16 a[2][kGBM * kGPadBf];
    bf16 b[2][kGBN * kGPadBf];
};
template <>
struct GemmSmem<float> {
    float a[2][kGBM * kGPadF];
    bf16 b[2][kGBN * kGPadBf];
};

template <typename AT>
__global__ void __launch_bounds__(256) gemm_tn_kernel(const AT* __restrict__ A, int M, int K,
                                                     const bf16* __restrict__ B0, int n0, float* __restrict__ C0,
                                                     int ldc0, const bf16* __restrict__ B1, int n1,
                                                     float* __restrict__ C1, int ldc1) {
    __shared__ __align__(16) GemmSmem<AT> sm;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
    const int wm = warp & 3, wn = warp >> 2;          // warp tile (32 rows, 32 outputs)
    const int m0 = blockIdx.x * kGBM, n0t = blockIdx.y * kGBN;
    const int N = n0 + n1;

    auto b_row = [&](int r) -> const bf16* {
        if (r < n0) return B0 + (int64_t)r * K;
        if (r < N) return B1 + (int64_t)(r - n0) * K;
        return nullptr;
    };
    auto stage = [&](int kt, int buf) {
        const int k0 = kt * kGBK;
        if constexpr (sizeof(AT) == 2) {
            // A: 128 rows x 64 B = 512 pieces of 16 B
            for (int i = tid; i < kGBM * 4; i += 256) {
                const int r = i >> 2, c = (i & 3) * 8;
                const bool ok = m0 + r < M;
                cp_async16(&sm.a[buf][r * kGPadBf + c], ok ? (const void*)(A + (int64_t)(m0 + r) * K + k0 + c) : (const void*)A,
                           ok ? 16 : 0);
            }
        } else {
            // A: 128 rows x 128 B = 1024 pieces of 16 B
            for (int i = tid; i < kGBM * 8; i += 256) {
                const int r = i >> 3, c = (i & 7) * 4;
                const bool ok = m0 + r < M;
                cp_async16(&sm.a[buf][r * kGPadF + c], ok ? (const void*)(A + (int64_t)(m0 + r) * K + k0 + c) : (const void*)A,
                           ok ? 16 : 0);
            }
        }
        // B: 64 rows x 64 B
        for (int i = tid; i < kGBN * 4; i += 256) {
            const int r = i >> 2, c = (i & 3) * 8;
            const bf16* br = b_row(n0t + r);
            cp_async16(&sm.b[buf][r * kGPadBf + c], br ? (const void*)(br + k0 + c) : (const void*)B0, br ? 16 : 0);
        }
        cp_async_commit();
    };

    float acc[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;

    griddep_wait();
    const int nk = K / kGBK;
    stage(0, 0);
    for (int kt = 0; kt < nk; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < nk) {
            stage(kt + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
#pragma unroll
        for (int ks = 0; ks < kGBK / 16; ++ks) {
            // B fragments: 4 n-tiles of 8 outputs, two per ldmatrix.x4
            // (matrices: tile j k-lo, tile j k-hi, tile j+1 k-lo, tile j+1 k-hi)
            uint32_t bfr[4][2];
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                const int r = wn * 32 + (j + (lane >> 4)) * 8 + (lane & 7);
                const int c = ks * 16 + ((lane >> 3) & 1) * 8;
                uint32_t t4[4];
                ldmatrix_x4(t4, &sm.b[buf][r * kGPadBf + c]);
                bfr[j][0] = t4[0];
                bfr[j][1] = t4[1];
                bfr[j + 1][0] = t4[2];
                bfr[j + 1][1] = t4[3];
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int rb = wm * 32 + i * 16;
                if constexpr (sizeof(AT) == 2) {
                    uint32_t afr[4];
                    const int r = rb + (lane & 15);
                    const int c = ks * 16 + (lane >> 4) * 8;
                    ldmatrix_x4(afr, &sm.a[buf][r * kGPadBf + c]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) mma_bf16_16816(acc[i][j], afr, bfr[j][0], bfr[j][1]);
                } else {
                    // fp32 A: rows g / g+8, channels 2tq.. / 2tq+8.. ; hi + lo pairs
                    const float* a0 = &sm.a[buf][(rb + g) * kGPadF + ks * 16 + 2 * tq];
                    const float* a1 = &sm.a[buf][(rb + g + 8) * kGPadF + ks * 16 + 2 * tq];
                    const float2 x00 = *reinterpret_cast<const float2*>(a0);
                    const float2 x10 = *reinterpret_cast<const float2*>(a1);
                    const float2 x01 = *reinterpret_cast<const float2*>(a0 + 8);
                    const float2 x11 = *reinterpret_cast<const float2*>(a1 + 8);
                    uint32_t hi[4], lo[4];
                    const float2 xs[4] = {x00, x10, x01, x11};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float h0 = __bfloat162float(__float2bfloat16_rn(xs[e].x));
                        const float h1 = __bfloat162float(__float2bfloat16_rn(xs[e].y));
                        hi[e] = pack_bf16(h0, h1);
                        lo[e] = pack_bf16(xs[e].x - h0, xs[e].y - h1);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        mma_bf16_16816(acc[i][j], hi, bfr[j][0], bfr[j][1]);
                        mma_bf16_16816(acc[i][j], lo, bfr[j][0], bfr[j][1]);
                    }
                }
            }
        }
        __syncthreads();   // the other buffer is refilled next iteration
    }
    // write C
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = m0 + wm * 32 + i * 16 + g + hh * 8;
                if (r >= M) continue;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int o = n0t + wn * 32 + j * 8 + 2 * tq + u;
                    const float v = acc[i][j][hh * 2 + u];
                    if (o < n0) C0[(int64_t)r * ldc0 + o] = v;
                    else if (o < N) C1[(int64_t)r * ldc1 + (o - n0)] = v;
                }
            }
        }
    }
    griddep_trigger();
}

// C0 [M][ldc0] (outputs 0..n0-1 from B0), C1 [M][ldc1] (outputs n0.. from B1).
// K must be a multiple of 32.
template <typename AT>
cudaError_t launch_gemm_tn(const AT* A, int M, int K, const bf16* B0, int n0, float* C0, int ldc0, const bf16* B1,
                           int n1, float* C1, int ldc1, cudaStream_t stream) {
    dim3 grid((M + kGBM - 1) / kGBM, (n0 + n1 + kGBN - 1) / kGBN);
    return launch_pdl(gemm_tn_kernel<AT>, grid, dim3(256), 0, stream, A, M, K, B0, n0, C0, ldc0, B1, n1, C1, ldc1);
}

template cudaError_t launch_gemm_tn<bf16>(const bf16*, int, int, const bf16*, int, float*, int, const bf16*, int, float*,
                                          int, cudaStream_t);
template cudaError_t launch_gemm_tn<float>(const float*, int, int, const bf16*, int, float*, int, const bf16*, int,
                                           float*, int, cudaStream_t);

}  // namespace csa
