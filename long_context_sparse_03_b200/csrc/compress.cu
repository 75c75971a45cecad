// compress.cu -- KV / indexer-key compression by m adjacent rows.
//
// DeepSeek-V4 summary (b-lab.team), "Core Methodological Innovations" 1:
// CSA compresses the KV cache by m "by combining adjacent entries"; HCA does
// the same with m' >> m.  Reading taken: a fixed per-position, per-channel
// weighted sum whose weights are a softmax over the m positions.
//
// Layout: one thread owns one 16-byte chunk (8 channels) of one output row,
// so a warp reads whole 256-byte (d = 128) or 128-byte (d = 64) raw rows with
// coalesced 128-bit loads, streaming m rows per output row.  The pooling
// weights are computed once per CTA into shared memory, before the wait on
// the preceding kernel (they depend only on the logits), and each CTA then
// loops over output rows: the grid is bounded by what the SMs hold at once,
// whatever block range is asked for.
#include <algorithm>

#include "common.cuh"

namespace csa {

// a_sh[i*D + c] = softmax over i of logits[i][c], for all 256 threads of the
// CTA: column c = t % D, part p = t / D of P = 256 / D; part p covers
// positions i = p, p + P, ...; red is 256 floats of scratch.
template <int D>
__device__ __forceinline__ void pool_weights_smem(const float* __restrict__ logits, int m, float* a_sh, float* red) {
    constexpr int P = 256 / D;
    const int t = threadIdx.x, c = t % D, p = t / D;
    for (int x = t; x < m * D; x += 256) a_sh[x] = logits[x];
    __syncthreads();
    float mx = -INFINITY;
    for (int i = p; i < m; i += P) mx = fmaxf(mx, a_sh[i * D + c]);
    red[t] = mx;
    __syncthreads();
    mx = red[c];
#pragma unroll
    for (int q = 1; q < P; ++q) mx = fmaxf(mx, red[q * D + c]);
    float s = 0.f;
    for (int i = p; i < m; i += P) {
        const float e = expf(a_sh[i * D + c] - mx);
        a_sh[i * D + c] = e;
        s += e;
    }
    __syncthreads();
    red[t] = s;
    __syncthreads();
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < P; ++q) sum += red[q * D + c];
    for (int i = p; i < m; i += P) a_sh[i * D + c] = a_sh[i * D + c] / sum;
    __syncthreads();
}

// Block range of sequence b (see csa_compress).
__device__ __forceinline__ void block_range(const int* lens, int b, int m, int blk_lo, int blk_hi, int& lo, int& hi) {
    const int nblk = lens[b] / m;
    if (blk_lo >= 0) {
        lo = blk_lo;
        hi = min(blk_hi, nblk);
    } else {
        lo = max(0, nblk - blk_hi);
        hi = nblk;
    }
}

// fp32 row (8 channels of one thread) -> bf16 row or E4M3 codes + scale.
// For E4M3 the TPR threads of a row are consecutive lanes of one warp.
template <int D, int FMT>
__device__ __forceinline__ void store_row(const float (&acc)[8], void* out, int64_t out_stride, float* out_scale,
                                          int64_t scale_stride, int b, int j, int chunk) {
    constexpr int TPR = D / 8;
    uint4 ob;
    uint32_t* obw = reinterpret_cast<uint32_t*>(&ob);
#pragma unroll
    for (int e = 0; e < 4; ++e) obw[e] = pack_bf16(acc[2 * e], acc[2 * e + 1]);   // round to nearest even
    if (FMT == 0) {
        bf16* dst = reinterpret_cast<bf16*>(out) + (int64_t)b * out_stride + (int64_t)j * D + chunk * 8;
        *reinterpret_cast<uint4*>(dst) = ob;
    } else {
        // E4M3 row with one fp32 scale: s = amax/448 of the bf16 row.
        float xv[8];
        const __nv_bfloat162* xb = reinterpret_cast<const __nv_bfloat162*>(&ob);
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(xb[e]);
            xv[2 * e] = f.x;
            xv[2 * e + 1] = f.y;
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
        const int lane = threadIdx.x & 31;
        const unsigned grp = (TPR >= 32 ? 0xffffffffu : ((1u << TPR) - 1u)) << (lane & ~(TPR - 1) & 31);
#pragma unroll
        for (int off = 1; off < TPR; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(grp, amax, off));
        const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        uint2 codes;
        uint16_t* cw = reinterpret_cast<uint16_t*>(&codes);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 pr = make_float2(__fdiv_rn(xv[2 * e], sc), __fdiv_rn(xv[2 * e + 1], sc));
            cw[e] = __nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
        }
        uint8_t* dst = reinterpret_cast<uint8_t*>(out) + (int64_t)b * out_stride + (int64_t)j * D + chunk * 8;
        *reinterpret_cast<uint2*>(dst) = codes;
        if (chunk == 0) out_scale[(int64_t)b * scale_stride + j] = sc;
    }
}

// acc += sum over i = i0, i0 + di, ... < m of a[i][chunk] * x_i[chunk], in order.
template <int D>
__device__ __forceinline__ void pool_chain(const bf16* __restrict__ src, const float* a_sh, int chunk, int i0, int di,
                                           int m, float (&acc)[8]) {
#pragma unroll 4
    for (int i = i0; i < m; i += di) {
        const uint4 v = ldg_stream(src + (int64_t)i * D);
        const float4 w0 = *reinterpret_cast<const float4*>(&a_sh[i * D + chunk * 8]);
        const float4 w1 = *reinterpret_cast<const float4*>(&a_sh[i * D + chunk * 8 + 4]);
        const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&v);
        const float2 x0 = __bfloat1622float2(x[0]), x1 = __bfloat1622float2(x[1]);
        const float2 x2 = __bfloat1622float2(x[2]), x3 = __bfloat1622float2(x[3]);
        acc[0] = fmaf(w0.x, x0.x, acc[0]);
        acc[1] = fmaf(w0.y, x0.y, acc[1]);
        acc[2] = fmaf(w0.z, x1.x, acc[2]);
        acc[3] = fmaf(w0.w, x1.y, acc[3]);
        acc[4] = fmaf(w1.x, x2.x, acc[4]);
        acc[5] = fmaf(w1.y, x2.y, acc[5]);
        acc[6] = fmaf(w1.z, x3.x, acc[6]);
        acc[7] = fmaf(w1.w, x3.y, acc[7]);
    }
}

// Light compression (m < kSplitM): RPC = 256 / (D/8) output rows per CTA
// pass, one fp32 FMA chain over i = 0..m-1 per output channel.
template <int D, int FMT>
__global__ void __launch_bounds__(256) compress_kernel(
    const bf16* __restrict__ raw, int64_t raw_stride, const int* __restrict__ lens, int m,
    const float* __restrict__ logits, int blk_lo, int blk_hi, void* __restrict__ out,
    int64_t out_stride, float* __restrict__ out_scale, int64_t scale_stride) {
    constexpr int TPR = D / 8;            // threads per output row
    constexpr int RPC = 256 / TPR;        // output rows per CTA pass
    extern __shared__ float a_sh[];       // [m][D] pooling weights, then 256 floats of scratch
    pool_weights_smem<D>(logits, m, a_sh, a_sh + (size_t)m * D);

    griddep_wait();
    const int b = blockIdx.y;
    int lo, hi;
    block_range(lens, b, m, blk_lo, blk_hi, lo, hi);
    const int chunk = threadIdx.x % TPR;
    for (int jb = lo + blockIdx.x * RPC; jb < hi; jb += gridDim.x * RPC) {
        const int j = jb + threadIdx.x / TPR;
        if (j >= hi) continue;
        const bf16* src = raw + (int64_t)b * raw_stride + (int64_t)j * m * D + chunk * 8;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        pool_chain<D>(src, a_sh, chunk, 0, 1, m, acc);
        store_row<D, FMT>(acc, out, out_stride, out_scale, scale_stride, b, j, chunk);
    }
    griddep_trigger();
}

// Heavy compression (m >= kSplitM): one output row per CTA pass; its 256
// threads are (16 position groups) x (D/8 channel chunks, D = 128) or (32
// groups) x (8 chunks, D = 64).  Group ig sums positions i = ig, ig + G, ...
// in order (one fp32 FMA chain each); the G chains are added in group order.
// The split only changes how the m products are grouped before rounding, and
// it is fixed by m (never by the batch).
constexpr int kSplitM = 16;

template <int D, int FMT>
__global__ void __launch_bounds__(256) compress_split_kernel(
    const bf16* __restrict__ raw, int64_t raw_stride, const int* __restrict__ lens, int m,
    const float* __restrict__ logits, int blk_lo, int blk_hi, void* __restrict__ out,
    int64_t out_stride, float* __restrict__ out_scale, int64_t scale_stride) {
    constexpr int TPR = D / 8;            // channel chunks
    constexpr int G = 256 / TPR;          // position groups
    extern __shared__ float a_sh[];       // [m][D] pooling weights, then [G][D] partial sums
    float* part = a_sh + (size_t)m * D;
    pool_weights_smem<D>(logits, m, a_sh, part);

    griddep_wait();
    const int b = blockIdx.y;
    int lo, hi;
    block_range(lens, b, m, blk_lo, blk_hi, lo, hi);
    const int chunk = threadIdx.x % TPR, ig = threadIdx.x / TPR;
    for (int j = lo + blockIdx.x; j < hi; j += gridDim.x) {   // uniform across the CTA
        const bf16* src = raw + (int64_t)b * raw_stride + (int64_t)j * m * D + chunk * 8;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        pool_chain<D>(src, a_sh, chunk, ig, G, m, acc);
#pragma unroll
        for (int e = 0; e < 8; ++e) part[ig * D + chunk * 8 + e] = acc[e];
        __syncthreads();
        if (threadIdx.x < TPR) {
            float r[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) r[e] = 0.f;
            for (int g2 = 0; g2 < G; ++g2)
#pragma unroll
                for (int e = 0; e < 8; ++e) r[e] += part[g2 * D + chunk * 8 + e];
            store_row<D, FMT>(r, out, out_stride, out_scale, scale_stride, b, j, chunk);
        }
        __syncthreads();   // part is rewritten by the next pass
    }
    griddep_trigger();
}

template <typename K>
static cudaError_t launch_bounded(K kern, size_t smem, int rows_per_pass, int span, int B, const bf16* raw,
                                  int64_t raw_stride, const int* lens, int m, const float* logits, int blk_lo,
                                  int blk_hi, void* out, int64_t out_stride, float* out_scale, int64_t scale_stride,
                                  cudaStream_t stream) {
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024) e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 256, smem) != cudaSuccess || occ <= 0) occ = 1;
    const int64_t resident = (int64_t)current_sm_count() * occ;
    const int64_t passes = ((int64_t)span + rows_per_pass - 1) / rows_per_pass;
    const int64_t gx = std::max<int64_t>(1, std::min<int64_t>(passes, resident / B));
    return launch_pdl(kern, dim3((unsigned)gx, (unsigned)B), dim3(256), smem, stream, raw, raw_stride, lens, m, logits,
                      blk_lo, blk_hi, out, out_stride, out_scale, scale_stride);
}

// Launch: grid.y = the sequences, grid.x = CTAs per sequence (at most what
// the SMs hold at once, divided among the sequences), each looping over rows.
cudaError_t launch_compress(const void* raw, int64_t raw_stride, const int* lens, int B, int d, int m,
                            const float* logits, int blk_lo, int blk_hi, void* out,
                            int64_t out_stride, int out_fmt, float* out_scale, int64_t scale_stride,
                            cudaStream_t stream) {
    const int span = blk_lo >= 0 ? (blk_hi - blk_lo) : blk_hi;
    if (span <= 0 || B <= 0) return cudaSuccess;
    const bf16* r = reinterpret_cast<const bf16*>(raw);
    const bool split = m >= kSplitM;
    const int tpr = d / 8;
    const size_t smem = sizeof(float) * ((size_t)m * d + (split ? (size_t)(256 / tpr) * d : 256));
    const int rpp = split ? 1 : 256 / tpr;
    cudaError_t e;
#define CSA_COMPRESS_GO(KERN) \
    launch_bounded(KERN, smem, rpp, span, B, r, raw_stride, lens, m, logits, blk_lo, blk_hi, out, out_stride, \
                   out_scale, scale_stride, stream)
    if (split) {
        if (d == 128) e = CSA_COMPRESS_GO((compress_split_kernel<128, 0>));
        else if (out_fmt == 0) e = CSA_COMPRESS_GO((compress_split_kernel<64, 0>));
        else e = CSA_COMPRESS_GO((compress_split_kernel<64, 1>));
    } else {
        if (d == 128) e = CSA_COMPRESS_GO((compress_kernel<128, 0>));
        else if (out_fmt == 0) e = CSA_COMPRESS_GO((compress_kernel<64, 0>));
        else e = CSA_COMPRESS_GO((compress_kernel<64, 1>));
    }
#undef CSA_COMPRESS_GO
    return e;
}

}  // namespace csa
