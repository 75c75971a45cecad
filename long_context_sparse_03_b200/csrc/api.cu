// api.cu -- the extern "C" boundary of libcsa (declared in include/csa.h).
//
// Validates every argument on the host before any launch (no side effects
// on error), lays out the caller's workspace, and launches the kernels of
// compress.cu, index_query.cu, index_score.cu and attend.cu on the caller's
// stream.  The library allocates no device memory.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/csa.h"
#include "common.cuh"

namespace csa {
cudaError_t launch_compress(const void* raw, int64_t raw_stride, const int* lens, int B, int d, int m,
                            const float* logits, int blk_lo, int blk_hi, void* out, int64_t out_stride,
                            int out_fmt, float* out_scale, int64_t scale_stride, cudaStream_t stream);
cudaError_t launch_index_query(const void* h, int T, int D, int r, int Hi, const void* W_dq, const void* W_uq,
                               const void* W_w, float* q_out, float* w_out, float* u_ws, cudaStream_t stream,
                               int* launches);
cudaError_t launch_index_score(const float* q, const float* w, const int* q_seq, const int* q_pos, int T, int Hi,
                               const void* kidx, int fmt, const float* kscale, int64_t kstride_elems, int64_t sstride,
                               int m, int max_blocks, int k, float* scores, int64_t ld_scores, unsigned* hist,
                               unsigned* cnt, unsigned* done, unsigned* thr, unsigned* status, cudaStream_t stream,
                               int* launches);
cudaError_t launch_index_select_tail(const float* scores, int64_t ld_scores, const unsigned* thr, const int* q_pos,
                                     int T, int m, int max_blocks, int k, uint64_t* cand, int64_t cand_cap,
                                     unsigned* cnt, int* out_idx, float* out_score, cudaStream_t stream,
                                     int* launches);
constexpr int kHistBins = 2048;
int attend_nsplit(int max_rows, bool dense);
cudaError_t launch_attend(const void* q, const int* q_seq, const int* q_pos, int T, int H, const void* comp,
                          int64_t comp_stride, const void* raw, int64_t raw_stride, int m, const int* idx, int k,
                          int max_blocks, int W, float scale, void* out, float* lse, float* part_o,
                          float* part_ml, unsigned* status, bool use_partials, cudaStream_t stream,
                          int* launches);
}  // namespace csa

namespace {

thread_local char g_err[512] = "";
std::atomic<uint64_t> g_launches{0};

csa_status fail(csa_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}
csa_status ok() {
    g_err[0] = 0;
    return CSA_OK;
}
csa_status cuda_fail(cudaError_t e, const char* where) {
    return fail(CSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}
void count(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

#define REQUIRE(cond, status, ...)               \
    do {                                         \
        if (!(cond)) return fail(status, __VA_ARGS__); \
    } while (0)

// ---------------------------------------------------------------- layouts
// candidate rows start 16-byte aligned (the rank pass stages them with cp.async)
int64_t cand_cap(int max_blocks) { return ((int64_t)max_blocks + 1) & ~(int64_t)1; }

struct IndexLayout {
    size_t hist, cnt, done, thr, scores, cand, q, w, u, total;
};
// header | hist [T][2048] | cnt [T] | done [T] | thr [T] | scores [T][max_blocks] fp32 |
// cand [T][cand_cap] u64 | q [T][Hi][64] | w [T][Hi] | u [T][r].
// The scoring pass zeroes the selection state (hist, cnt, done: contiguous)
// itself.  csa_index_query keeps u at the very end of whatever workspace it
// is given.
// Row stride of the workspace score matrix: a multiple of 4 floats, so every
// row starts 16-byte aligned (the collect pass reads it 16 bytes at a time).
int64_t score_ld(int max_blocks) { return ((int64_t)max_blocks + 3) & ~(int64_t)3; }

IndexLayout index_layout(int T, int r, int Hi, int max_blocks) {
    IndexLayout L;
    size_t off = CSA_WS_HEADER_BYTES;
    L.hist = off;
    L.cnt = off + (size_t)T * csa::kHistBins * 4;
    L.done = L.cnt + (size_t)T * 4;
    L.thr = L.done + (size_t)T * 4;
    off = up256(L.thr + (size_t)T * 4);
    L.scores = off;
    off = up256(off + (size_t)T * score_ld(max_blocks) * 4);
    L.cand = off;
    off = up256(off + (size_t)T * cand_cap(max_blocks) * 8);
    L.q = off;
    off = up256(off + (size_t)T * Hi * 64 * 4);
    L.w = off;
    off = up256(off + (size_t)T * Hi * 4);
    L.u = off;
    off = up256(off + (size_t)T * r * 4);
    L.total = off;
    return L;
}

struct AttendLayout {
    size_t part_o, part_ml, total;
};
AttendLayout attend_layout(int T, int H, int max_rows, bool dense) {
    AttendLayout L;
    const int ns = csa::attend_nsplit(max_rows, dense);
    size_t off = CSA_WS_HEADER_BYTES;
    L.part_o = off;
    off = up256(off + (size_t)T * ns * H * 128 * 4);
    L.part_ml = off;
    off = up256(off + (size_t)T * ns * H * 2 * 4);
    L.total = off;
    return L;
}

csa_status check_index_common(const float* q, const float* w, const int32_t* q_seq, const int32_t* q_pos, int T,
                              int Hi, const void* kidx, int kidx_fmt, const float* kidx_scale,
                              int64_t kidx_seq_stride, int64_t scale_seq_stride, int m, int max_blocks) {
    REQUIRE(T >= 0, CSA_ERR_SHAPE, "T = %d < 0", T);
    REQUIRE(T <= CSA_MAX_T, CSA_ERR_UNSUPPORTED, "T = %d > %d", T, CSA_MAX_T);
    REQUIRE(Hi >= 1 && Hi <= CSA_MAX_HI, CSA_ERR_UNSUPPORTED, "Hi = %d outside 1..%d", Hi, CSA_MAX_HI);
    REQUIRE(m >= 1 && m <= CSA_MAX_M, CSA_ERR_UNSUPPORTED, "m = %d outside 1..%d", m, CSA_MAX_M);
    REQUIRE(max_blocks >= 1, CSA_ERR_SHAPE, "max_blocks = %d < 1", max_blocks);
    REQUIRE(kidx_fmt == CSA_FMT_BF16 || kidx_fmt == CSA_FMT_FP8E4M3, CSA_ERR_UNSUPPORTED, "kidx_fmt = %d", kidx_fmt);
    if (T == 0) return ok();
    REQUIRE(q && w && q_seq && q_pos && kidx, CSA_ERR_NULL, "q, w, q_seq, q_pos and kidx are required");
    REQUIRE(kidx_fmt == CSA_FMT_BF16 || kidx_scale, CSA_ERR_NULL, "E4M3 keys need kidx_scale");
    REQUIRE(kidx_seq_stride >= 0 && scale_seq_stride >= 0, CSA_ERR_SHAPE, "negative stride");
    REQUIRE(aligned16(kidx) && aligned16(q), CSA_ERR_ALIGN, "kidx and q must be 16-byte aligned");
    REQUIRE(kidx_seq_stride % (kidx_fmt == CSA_FMT_BF16 ? 8 : 16) == 0, CSA_ERR_ALIGN,
            "kidx_seq_stride must keep rows 16-byte aligned");
    return ok();
}

}  // namespace

extern "C" {

const char* csa_status_string(csa_status s) {
    switch (s) {
        case CSA_OK: return "CSA_OK";
        case CSA_ERR_NULL: return "CSA_ERR_NULL";
        case CSA_ERR_SHAPE: return "CSA_ERR_SHAPE";
        case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
        case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE";
        case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
        case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT";
        case CSA_ERR_DEVICE: return "CSA_ERR_DEVICE";
        case CSA_ERR_ALIGN: return "CSA_ERR_ALIGN";
    }
    return "CSA_ERR_UNKNOWN";
}

const char* csa_last_error(void) { return g_err; }

uint64_t csa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

csa_status csa_workspace_init(void* ws, size_t ws_bytes, csa_stream_t stream) {
    REQUIRE(ws, CSA_ERR_NULL, "ws is NULL");
    REQUIRE(ws_bytes >= CSA_WS_HEADER_BYTES, CSA_ERR_WORKSPACE, "workspace smaller than its header");
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "csa_workspace_init");
    return ok();
}

csa_status csa_status_check(void* ws, size_t ws_bytes, csa_stream_t stream) {
    REQUIRE(ws, CSA_ERR_NULL, "ws is NULL");
    REQUIRE(ws_bytes >= CSA_WS_HEADER_BYTES, CSA_ERR_WORKSPACE, "workspace smaller than its header");
    unsigned word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(word), (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "csa_status_check");
    if (word & CSA_DEV_TIMEOUT) return fail(CSA_ERR_TIMEOUT, "device wait timed out (status 0x%x)", word);
    if (word) return fail(CSA_ERR_DEVICE, "device status bits 0x%x (1 = out-of-range block index)", word);
    return ok();
}

// ---------------------------------------------------------------- compress
csa_status csa_compress(const void* raw, int64_t raw_seq_stride, const int32_t* lens, int B, int d, int m,
                        const float* pool_logits, int blk_lo, int blk_hi, void* out, int64_t out_seq_stride,
                        int out_fmt, float* out_scale, int64_t scale_seq_stride, csa_stream_t stream) {
    REQUIRE(B >= 0, CSA_ERR_SHAPE, "B = %d < 0", B);
    REQUIRE(B <= CSA_MAX_T, CSA_ERR_UNSUPPORTED, "B = %d > %d", B, CSA_MAX_T);
    REQUIRE(d == 64 || d == 128, CSA_ERR_UNSUPPORTED, "d = %d (64 or 128)", d);
    REQUIRE(m >= 1 && m <= CSA_MAX_M, CSA_ERR_UNSUPPORTED, "m = %d outside 1..%d", m, CSA_MAX_M);
    REQUIRE(out_fmt == CSA_FMT_BF16 || (out_fmt == CSA_FMT_FP8E4M3 && d == 64), CSA_ERR_UNSUPPORTED,
            "out_fmt %d with d = %d (E4M3 only for d = 64)", out_fmt, d);
    REQUIRE(blk_lo >= -1, CSA_ERR_SHAPE, "blk_lo = %d < -1", blk_lo);
    REQUIRE(blk_lo < 0 ? blk_hi >= 0 : blk_hi >= blk_lo, CSA_ERR_SHAPE, "bad block range [%d, %d)", blk_lo, blk_hi);
    REQUIRE(raw_seq_stride >= 0 && out_seq_stride >= 0 && scale_seq_stride >= 0, CSA_ERR_SHAPE, "negative stride");
    if (B == 0 || (blk_lo >= 0 ? blk_hi == blk_lo : blk_hi == 0)) return ok();
    REQUIRE(raw && lens && pool_logits && out, CSA_ERR_NULL, "raw, lens, pool_logits and out are required");
    REQUIRE(out_fmt == CSA_FMT_BF16 || out_scale, CSA_ERR_NULL, "E4M3 output needs out_scale");
    REQUIRE(aligned16(raw) && aligned16(out), CSA_ERR_ALIGN, "raw and out must be 16-byte aligned");
    REQUIRE(raw_seq_stride % 8 == 0, CSA_ERR_ALIGN, "raw_seq_stride must be a multiple of 8");
    REQUIRE(out_seq_stride % (out_fmt == CSA_FMT_BF16 ? 8 : 16) == 0, CSA_ERR_ALIGN,
            "out_seq_stride must keep rows 16-byte aligned");
    cudaError_t e = csa::launch_compress(raw, raw_seq_stride, lens, B, d, m, pool_logits, blk_lo, blk_hi, out,
                                         out_seq_stride, out_fmt, out_scale, scale_seq_stride,
                                         (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "csa_compress");
    count(1);
    return ok();
}

// ---------------------------------------------------------------- indexer
size_t csa_index_workspace_size(int T, int r, int Hi, int k, int max_blocks) {
    (void)k;
    if (T < 0 || r < 0 || Hi < 0 || max_blocks < 0) return 0;
    return index_layout(T, r, Hi, max_blocks).total;
}

csa_status csa_index_query(const void* h, int T, int D, int r, int Hi, const void* W_dq, const void* W_uq,
                           const void* W_w, float* q_out, float* w_out, void* ws, size_t ws_bytes,
                           csa_stream_t stream) {
    REQUIRE(T >= 0 && D >= 8 && r >= 8, CSA_ERR_SHAPE, "T = %d, D = %d, r = %d", T, D, r);
    REQUIRE(D % 8 == 0 && r % 8 == 0, CSA_ERR_UNSUPPORTED, "D and r must be multiples of 8");
    REQUIRE(D <= CSA_MAX_D && r <= CSA_MAX_D, CSA_ERR_UNSUPPORTED, "D and r must be <= %d", CSA_MAX_D);
    REQUIRE(Hi >= 1 && Hi <= CSA_MAX_HI, CSA_ERR_UNSUPPORTED, "Hi = %d outside 1..%d", Hi, CSA_MAX_HI);
    if (T == 0) return ok();
    REQUIRE(h && W_dq && W_uq && W_w && q_out && w_out && ws, CSA_ERR_NULL, "a required pointer is NULL");
    REQUIRE(aligned16(h) && aligned16(W_dq) && aligned16(W_uq) && aligned16(W_w) && aligned16(ws), CSA_ERR_ALIGN,
            "h, weights and ws must be 16-byte aligned");
    const size_t ubytes = up256((size_t)T * r * 4);
    const size_t need = CSA_WS_HEADER_BYTES + ubytes;
    REQUIRE(ws_bytes >= need, CSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
    // u lives at the end of the workspace (256-byte aligned), clear of the
    // selection state at its start
    const size_t uoff = (ws_bytes - ubytes) & ~(size_t)255;
    int n = 0;
    cudaError_t e = csa::launch_index_query(h, T, D, r, Hi, W_dq, W_uq, W_w, q_out, w_out,
                                            reinterpret_cast<float*>((char*)ws + uoff), (cudaStream_t)stream, &n);
    count(n);
    if (e != cudaSuccess) return cuda_fail(e, "csa_index_query");
    return ok();
}

csa_status csa_index_scores(const float* q, const float* w, const int32_t* q_seq, const int32_t* q_pos, int T,
                            int Hi, const void* kidx, int kidx_fmt, const float* kidx_scale,
                            int64_t kidx_seq_stride, int64_t scale_seq_stride, int m, int max_blocks, float* scores,
                            csa_stream_t stream) {
    csa_status s = check_index_common(q, w, q_seq, q_pos, T, Hi, kidx, kidx_fmt, kidx_scale, kidx_seq_stride,
                                      scale_seq_stride, m, max_blocks);
    if (s != CSA_OK || T == 0) return s;
    REQUIRE(scores, CSA_ERR_NULL, "scores is NULL");
    // invisible entries stay NaN (all-ones bytes)
    cudaError_t e = cudaMemsetAsync(scores, 0xFF, (size_t)T * max_blocks * 4, (cudaStream_t)stream);
    int n = 0;
    if (e == cudaSuccess)
        e = csa::launch_index_score(q, w, q_seq, q_pos, T, Hi, kidx, kidx_fmt, kidx_scale, kidx_seq_stride,
                                    scale_seq_stride, m, max_blocks, 1, scores, max_blocks, nullptr, nullptr,
                                    nullptr, nullptr, nullptr, (cudaStream_t)stream, &n);
    count(n);
    if (e != cudaSuccess) return cuda_fail(e, "csa_index_scores");
    return ok();
}

static csa_status stage_score(const char* who, const float* q, const float* w, const int32_t* q_seq,
                              const int32_t* q_pos, int T, int Hi, const void* kidx, int kidx_fmt,
                              const float* kidx_scale, int64_t kidx_seq_stride, int64_t scale_seq_stride, int m,
                              int max_blocks, int k, const IndexLayout& L, void* ws, cudaStream_t stream) {
    char* base = (char*)ws;
    int n = 0;
    cudaError_t e = csa::launch_index_score(q, w, q_seq, q_pos, T, Hi, kidx, kidx_fmt, kidx_scale, kidx_seq_stride,
                                            scale_seq_stride, m, max_blocks, k,
                                            reinterpret_cast<float*>(base + L.scores), score_ld(max_blocks),
                                            reinterpret_cast<unsigned*>(base + L.hist),
                                            reinterpret_cast<unsigned*>(base + L.cnt),
                                            reinterpret_cast<unsigned*>(base + L.done),
                                            reinterpret_cast<unsigned*>(base + L.thr), reinterpret_cast<unsigned*>(base),
                                            stream, &n);
    count(n);
    if (e != cudaSuccess) return cuda_fail(e, who);
    return ok();
}

static csa_status stage_merge(const char* who, const int32_t* q_pos, int T, int m, int max_blocks, int k,
                              int32_t* out_idx, float* out_score, const IndexLayout& L, void* ws,
                              cudaStream_t stream) {
    char* base = (char*)ws;
    int n = 0;
    cudaError_t e = csa::launch_index_select_tail(
        reinterpret_cast<const float*>(base + L.scores), score_ld(max_blocks), reinterpret_cast<const unsigned*>(base + L.thr),
        q_pos, T, m, max_blocks, k, reinterpret_cast<uint64_t*>(base + L.cand), cand_cap(max_blocks),
        reinterpret_cast<unsigned*>(base + L.cnt), out_idx, out_score, stream, &n);
    count(n);
    if (e != cudaSuccess) return cuda_fail(e, who);
    return ok();
}

csa_status csa_index_stage_score(const float* q, const float* w, const int32_t* q_seq, const int32_t* q_pos, int T,
                                 int Hi, const void* kidx, int kidx_fmt, const float* kidx_scale,
                                 int64_t kidx_seq_stride, int64_t scale_seq_stride, int m, int max_blocks, int k,
                                 void* ws, size_t ws_bytes, csa_stream_t stream) {
    csa_status s = check_index_common(q, w, q_seq, q_pos, T, Hi, kidx, kidx_fmt, kidx_scale, kidx_seq_stride,
                                      scale_seq_stride, m, max_blocks);
    if (s != CSA_OK) return s;
    REQUIRE(k >= 1 && k <= CSA_MAX_K, CSA_ERR_UNSUPPORTED, "k = %d outside 1..%d", k, CSA_MAX_K);
    if (T == 0) return ok();
    REQUIRE(ws, CSA_ERR_WORKSPACE, "ws is NULL");
    REQUIRE(aligned16(ws), CSA_ERR_ALIGN, "ws must be 16-byte aligned");
    IndexLayout L = index_layout(T, 0, 0, max_blocks);
    REQUIRE(ws_bytes >= L.total, CSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    return stage_score("csa_index_stage_score", q, w, q_seq, q_pos, T, Hi, kidx, kidx_fmt, kidx_scale,
                       kidx_seq_stride, scale_seq_stride, m, max_blocks, k, L, ws, (cudaStream_t)stream);
}

csa_status csa_index_stage_merge(const int32_t* q_pos, int T, int m, int max_blocks, int k, int32_t* out_idx,
                                 float* out_score, void* ws, size_t ws_bytes, csa_stream_t stream) {
    REQUIRE(T >= 0 && max_blocks >= 1, CSA_ERR_SHAPE, "T = %d, max_blocks = %d", T, max_blocks);
    REQUIRE(T <= CSA_MAX_T, CSA_ERR_UNSUPPORTED, "T = %d > %d", T, CSA_MAX_T);
    REQUIRE(m >= 1 && m <= CSA_MAX_M, CSA_ERR_UNSUPPORTED, "m = %d outside 1..%d", m, CSA_MAX_M);
    REQUIRE(k >= 1 && k <= CSA_MAX_K, CSA_ERR_UNSUPPORTED, "k = %d outside 1..%d", k, CSA_MAX_K);
    if (T == 0) return ok();
    REQUIRE(q_pos && out_idx, CSA_ERR_NULL, "q_pos and out_idx are required");
    REQUIRE(ws, CSA_ERR_WORKSPACE, "ws is NULL");
    IndexLayout L = index_layout(T, 0, 0, max_blocks);
    REQUIRE(ws_bytes >= L.total, CSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    return stage_merge("csa_index_stage_merge", q_pos, T, m, max_blocks, k, out_idx, out_score, L, ws,
                       (cudaStream_t)stream);
}

csa_status csa_index_select(const float* q, const float* w, const int32_t* q_seq, const int32_t* q_pos, int T,
                            int Hi, const void* kidx, int kidx_fmt, const float* kidx_scale, int64_t kidx_seq_stride,
                            int64_t scale_seq_stride, int m, int max_blocks, int k, int32_t* out_idx,
                            float* out_score, void* ws, size_t ws_bytes, csa_stream_t stream) {
    REQUIRE(T == 0 || out_idx, CSA_ERR_NULL, "out_idx is NULL");
    csa_status s = csa_index_stage_score(q, w, q_seq, q_pos, T, Hi, kidx, kidx_fmt, kidx_scale, kidx_seq_stride,
                                         scale_seq_stride, m, max_blocks, k, ws, ws_bytes, stream);
    if (s != CSA_OK) return s;
    return csa_index_stage_merge(q_pos, T, m, max_blocks, k, out_idx, out_score, ws, ws_bytes, stream);
}

csa_status csa_index_topk(const void* h, int D, int r, const void* W_dq, const void* W_uq, const void* W_w,
                          const int32_t* q_seq, const int32_t* q_pos, int T, int Hi, const void* kidx, int kidx_fmt,
                          const float* kidx_scale, int64_t kidx_seq_stride, int64_t scale_seq_stride, int m,
                          int max_blocks, int k, int32_t* out_idx, float* out_score, void* ws, size_t ws_bytes,
                          csa_stream_t stream) {
    REQUIRE(T >= 0, CSA_ERR_SHAPE, "T = %d < 0", T);
    REQUIRE(T <= CSA_MAX_T, CSA_ERR_UNSUPPORTED, "T = %d > %d", T, CSA_MAX_T);
    REQUIRE(Hi >= 1 && Hi <= CSA_MAX_HI, CSA_ERR_UNSUPPORTED, "Hi = %d outside 1..%d", Hi, CSA_MAX_HI);
    REQUIRE(r >= 0, CSA_ERR_SHAPE, "r = %d < 0", r);
    REQUIRE(k >= 1 && k <= CSA_MAX_K, CSA_ERR_UNSUPPORTED, "k = %d outside 1..%d", k, CSA_MAX_K);
    REQUIRE(max_blocks >= 1, CSA_ERR_SHAPE, "max_blocks = %d < 1", max_blocks);
    if (T == 0) return ok();
    REQUIRE(out_idx, CSA_ERR_NULL, "out_idx is NULL");
    REQUIRE(ws, CSA_ERR_WORKSPACE, "ws is NULL");
    IndexLayout L = index_layout(T, r, Hi, max_blocks);
    REQUIRE(ws_bytes >= L.total, CSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    float* qb = reinterpret_cast<float*>((char*)ws + L.q);
    float* wb = reinterpret_cast<float*>((char*)ws + L.w);
    csa_status c = check_index_common(qb, wb, q_seq, q_pos, T, Hi, kidx, kidx_fmt, kidx_scale, kidx_seq_stride,
                                      scale_seq_stride, m, max_blocks);
    if (c != CSA_OK) return c;
    csa_status s = csa_index_query(h, T, D, r, Hi, W_dq, W_uq, W_w, qb, wb, ws, ws_bytes, stream);
    if (s != CSA_OK) return s;
    s = stage_score("csa_index_topk", qb, wb, q_seq, q_pos, T, Hi, kidx, kidx_fmt, kidx_scale, kidx_seq_stride,
                    scale_seq_stride, m, max_blocks, k, L, ws, (cudaStream_t)stream);
    if (s != CSA_OK) return s;
    return stage_merge("csa_index_topk", q_pos, T, m, max_blocks, k, out_idx, out_score, L, ws,
                       (cudaStream_t)stream);
}

// ---------------------------------------------------------------- attention
size_t csa_attend_workspace_size(int T, int H, int max_rows) {
    if (T < 0 || H < 0 || max_rows < 0) return 0;
    return attend_layout(T, H, max_rows, false).total;
}

size_t hca_attend_workspace_size(int T, int H, int max_rows) {
    if (T < 0 || H < 0 || max_rows < 0) return 0;
    return attend_layout(T, H, max_rows, true).total;
}

static csa_status attend_common(const char* who, const void* q, const int32_t* q_seq, const int32_t* q_pos, int T,
                                int H, const void* comp, int64_t comp_seq_stride, const void* raw,
                                int64_t raw_seq_stride, int m, const int32_t* idx, int k, int max_blocks, int W,
                                float scale, void* out, float* lse, void* ws, size_t ws_bytes,
                                csa_stream_t stream) {
    REQUIRE(T >= 0, CSA_ERR_SHAPE, "T = %d < 0", T);
    REQUIRE(T <= CSA_MAX_T, CSA_ERR_UNSUPPORTED, "T = %d > %d", T, CSA_MAX_T);
    REQUIRE(H >= 16 && H <= 128 && H % 16 == 0, CSA_ERR_UNSUPPORTED, "H = %d (16..128, multiple of 16)", H);
    REQUIRE(m >= 1 && m <= CSA_MAX_M, CSA_ERR_UNSUPPORTED, "m = %d outside 1..%d", m, CSA_MAX_M);
    REQUIRE(W >= 0 && W <= CSA_MAX_W, CSA_ERR_UNSUPPORTED, "W = %d outside 0..%d", W, CSA_MAX_W);
    REQUIRE(std::isfinite(scale), CSA_ERR_SHAPE, "scale is not finite");
    REQUIRE(comp_seq_stride >= 0 && raw_seq_stride >= 0, CSA_ERR_SHAPE, "negative stride");
    if (T == 0) return ok();
    REQUIRE(q && q_seq && q_pos && comp && raw && out, CSA_ERR_NULL, "q, q_seq, q_pos, comp, raw, out are required");
    REQUIRE(aligned16(q) && aligned16(comp) && aligned16(raw), CSA_ERR_ALIGN, "q, comp and raw must be 16-byte aligned");
    REQUIRE(comp_seq_stride % 8 == 0 && raw_seq_stride % 8 == 0, CSA_ERR_ALIGN, "strides must be multiples of 8");
    REQUIRE(ws, CSA_ERR_WORKSPACE, "ws is NULL");
    REQUIRE(aligned16(ws), CSA_ERR_ALIGN, "ws must be 16-byte aligned");
    const int max_rows = (idx ? k : max_blocks) + W;
    AttendLayout L = attend_layout(T, H, max_rows, idx == nullptr);
    REQUIRE(ws_bytes >= L.total, CSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    int n = 0;
    cudaError_t e = csa::launch_attend(q, q_seq, q_pos, T, H, comp, comp_seq_stride, raw, raw_seq_stride, m, idx, k,
                                       max_blocks, W, scale, out, lse,
                                       reinterpret_cast<float*>((char*)ws + L.part_o),
                                       reinterpret_cast<float*>((char*)ws + L.part_ml),
                                       reinterpret_cast<unsigned*>(ws), false, (cudaStream_t)stream, &n);
    count(n);
    if (e != cudaSuccess) return cuda_fail(e, who);
    return ok();
}

csa_status csa_sparse_attend(const void* q, const int32_t* q_seq, const int32_t* q_pos, int T, int H,
                             const void* comp, int64_t comp_seq_stride, const void* raw, int64_t raw_seq_stride,
                             int m, const int32_t* idx, int k, int W, float scale, void* out, float* lse, void* ws,
                             size_t ws_bytes, csa_stream_t stream) {
    REQUIRE(k >= 1 && k <= CSA_MAX_K, CSA_ERR_UNSUPPORTED, "k = %d outside 1..%d", k, CSA_MAX_K);
    REQUIRE(T == 0 || idx, CSA_ERR_NULL, "idx is NULL");
    return attend_common("csa_sparse_attend", q, q_seq, q_pos, T, H, comp, comp_seq_stride, raw, raw_seq_stride, m,
                         idx, k, 0, W, scale, out, lse, ws, ws_bytes, stream);
}

csa_status hca_attend(const void* q, const int32_t* q_seq, const int32_t* q_pos, int T, int H, const void* comp,
                      int64_t comp_seq_stride, const void* raw, int64_t raw_seq_stride, int m, int max_blocks, int W,
                      float scale, void* out, float* lse, void* ws, size_t ws_bytes, csa_stream_t stream) {
    REQUIRE(max_blocks >= 0, CSA_ERR_SHAPE, "max_blocks = %d < 0", max_blocks);
    return attend_common("hca_attend", q, q_seq, q_pos, T, H, comp, comp_seq_stride, raw, raw_seq_stride, m, nullptr,
                         0, max_blocks, W, scale, out, lse, ws, ws_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------- attention without allocation
// csa_sparse_attend_noalloc: the same attention as csa_sparse_attend, with its
// split-K scratch in a fixed array of device memory that belongs to the
// library instead of a caller-supplied workspace.  For callers that may not
// allocate device memory at all (see include/csa.h).
constexpr size_t kNoAllocScratchBytes = CSA_NOALLOC_SCRATCH_BYTES;   // 16 MiB on every GPU that loads the library
static __device__ __align__(256) unsigned char g_attend_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[256];   // device address of g_attend_scratch, per device ordinal

// The host-side name g_attend_scratch is only a stand-in for the array; its
// device address is looked up once per device, with that device current.
csa_status scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "csa_sparse_attend_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= 256) return fail(CSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attend_scratch);
        if (e != cudaSuccess || !p) return cuda_fail(e, "csa_sparse_attend_noalloc: cudaGetSymbolAddress");
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return CSA_OK;
}
}  // namespace

extern "C" {

csa_status csa_sparse_attend_noalloc(const void* q, const int32_t* q_seq, const int32_t* q_pos, int T, int H,
                                     const void* comp, int64_t comp_seq_stride, const void* raw,
                                     int64_t raw_seq_stride, int m, const int32_t* idx, int k, int W, float scale,
                                     void* out, float* lse, csa_stream_t stream) {
    REQUIRE(k >= 1 && k <= CSA_MAX_K, CSA_ERR_UNSUPPORTED, "k = %d outside 1..%d", k, CSA_MAX_K);
    REQUIRE(T >= 0, CSA_ERR_SHAPE, "T = %d < 0", T);
    REQUIRE(T <= CSA_MAX_T, CSA_ERR_UNSUPPORTED, "T = %d > %d", T, CSA_MAX_T);
    REQUIRE(H >= 16 && H <= 128 && H % 16 == 0, CSA_ERR_UNSUPPORTED, "H = %d (16..128, multiple of 16)", H);
    REQUIRE(m >= 1 && m <= CSA_MAX_M, CSA_ERR_UNSUPPORTED, "m = %d outside 1..%d", m, CSA_MAX_M);
    REQUIRE(W >= 0 && W <= CSA_MAX_W, CSA_ERR_UNSUPPORTED, "W = %d outside 0..%d", W, CSA_MAX_W);
    REQUIRE(std::isfinite(scale), CSA_ERR_SHAPE, "scale is not finite");
    REQUIRE(comp_seq_stride >= 0 && raw_seq_stride >= 0, CSA_ERR_SHAPE, "negative stride");
    if (T == 0) return ok();
    REQUIRE(q && q_seq && q_pos && comp && raw && out && idx, CSA_ERR_NULL,
            "q, q_seq, q_pos, comp, raw, idx and out are required");
    REQUIRE(aligned16(q) && aligned16(comp) && aligned16(raw), CSA_ERR_ALIGN, "q, comp and raw must be 16-byte aligned");
    REQUIRE(comp_seq_stride % 8 == 0 && raw_seq_stride % 8 == 0, CSA_ERR_ALIGN, "strides must be multiples of 8");
    const AttendLayout L = attend_layout(T, H, k + W, false);
    REQUIRE(L.total <= kNoAllocScratchBytes, CSA_ERR_WORKSPACE,
            "this call needs %zu bytes of scratch; the fixed scratch holds %zu (use csa_sparse_attend with a "
            "workspace for larger T, H, k + W)",
            L.total, kNoAllocScratchBytes);
    void* base = nullptr;
    csa_status s = scratch_address(&base);
    if (s != CSA_OK) return s;
    int n = 0;
    cudaError_t e = csa::launch_attend(q, q_seq, q_pos, T, H, comp, comp_seq_stride, raw, raw_seq_stride, m, idx, k,
                                       0, W, scale, out, lse, reinterpret_cast<float*>((char*)base + L.part_o),
                                       reinterpret_cast<float*>((char*)base + L.part_ml), nullptr, true,
                                       (cudaStream_t)stream, &n);
    count(n);
    if (e != cudaSuccess) return cuda_fail(e, "csa_sparse_attend_noalloc");
    return ok();
}

}  // extern "C"
