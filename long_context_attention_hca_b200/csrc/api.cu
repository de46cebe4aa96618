// api.cu -- extern "C" entry points: argument validation, then the launch.
// Every check happens on the host before any work is queued, so a rejected
// call leaves the stream untouched.  See include/hca.h for the contract.
#include <mutex>

#include <atomic>

#include "common.cuh"

namespace hca {

int compress_launch(int m, const uint16_t* x, const uint16_t* gate, int64_t seq_stride,
                    const float* bias, int B, int64_t n_blocks, const hca_kv_layout& L,
                    const hca_kv_cache& out, int64_t entry_begin, const hca_entry_extras* ex, cudaStream_t st);
int token_prep_launch(const uint16_t* x, const int32_t* pos, int64_t n, const hca_kv_layout& L,
                      const hca_entry_extras* ex, uint16_t* out, cudaStream_t st);
int state_append_launch(const uint16_t* x, const uint16_t* gate, const uint16_t* win_x, int B, int d, int64_t pos,
                        uint16_t* window, int W, uint16_t* tail_x, uint16_t* tail_gate, int m, cudaStream_t st);
int overlap_launch(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                   const uint16_t* a_prev, const uint16_t* za_prev, int64_t seq_stride, const float* bias, int B,
                   int64_t n_blocks, int D, int d_rope, int g, uint8_t* codes, float* scales, uint16_t* rope,
                   uint8_t* k_sf, int64_t cap, int64_t entry_begin, bool key, cudaStream_t st);
int index_launch(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                 const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                 int B, int Tq, int64_t Nc_cap, int Hi, int c, int m, void* scores, cudaStream_t st, bool bf16);
int topk_launch(const float* scores, const int32_t* q_pos, int R, int64_t Nc_cap, int m, int k,
                int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, cudaStream_t st);
bool topk_wide_preferred(int R, int64_t Nc_cap);
size_t topk_wide_ws_bytes(int R, int64_t Nc_cap);
int topk_wide_clear(void* ws, int R, int64_t Nc_cap, cudaStream_t st);
uint32_t* topk_wide_hist(void* ws, int64_t Nc_cap, int64_t* stride_u32);
int topk_wide_select(const void* scores, const int32_t* q_pos, int R, int64_t Nc_cap, int m, int k,
                     int32_t* idx, int32_t* count, void* ws, cudaStream_t st, bool bf16);
int topk_wide_launch(const void* scores, const int32_t* q_pos, int R, int64_t Nc_cap, int m, int k,
                     int32_t* idx, int32_t* count, void* ws, cudaStream_t st, bool bf16);
int index_launch_hist(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                      const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                      int B, int64_t Nc_cap, int Hi, int c, int m, void* scores, uint32_t* hist,
                      int64_t hist_stride, cudaStream_t st, bool bf16);
size_t decode_ws_bytes(int B, int H, int D, int max_comp, int W);
int attn_decode_launch(const uint16_t* q, int B, int H, const hca_kv_layout& L, const hca_kv_cache& kv,
                       const int32_t* idx, int idx_stride, const int32_t* n_comp, int max_comp,
                       const uint16_t* window, int W, float softmax_scale, const hca_attn_extras* ex,
                       uint16_t* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t st);
int attn_prefill_launch(const uint16_t* q, int Tq, int H, int p0, int m, const hca_kv_layout& L,
                        const hca_kv_cache& kv, const int32_t* idx, int idx_stride, const int32_t* count,
                        const uint16_t* raw, int W, float softmax_scale, const hca_attn_extras* ex,
                        uint16_t* out, cudaStream_t st);

int tc_take_device_error();
int index_take_device_error();

static thread_local int g_last_cuda_error = 0;
void set_last_cuda_error(int e) { g_last_cuda_error = e; }

int sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

namespace {

bool layout_ok(const hca_kv_layout& L) {
    return (L.d == 512 && L.d_rope == 64 && L.scale_group == 64) ||
           (L.d == 128 && L.d_rope == 32 && L.scale_group == 32);
}

bool cache_ptrs_ok(const hca_kv_cache& c) {
    return c.codes && c.scales && c.rope && aligned16(c.codes) && aligned16(c.scales) && aligned16(c.rope) &&
           c.capacity >= 0;
}

#define REQUIRE(cond) do { if (!(cond)) return HCA_ERR_INVALID_ARG; } while (0)
#define REQ_PTR(p) REQUIRE((p) != nullptr && aligned16(p))

bool entry_extras_ok(const hca_entry_extras* ex) {
    if (!ex) return true;
    if (ex->norm_w && !aligned16(ex->norm_w)) return false;
    if (ex->inv_freq && !aligned16(ex->inv_freq)) return false;
    return ex->norm_eps >= 0.0f;
}

bool attn_extras_ok(const hca_attn_extras* ex, bool decode) {
    if (!ex) return true;
    if (ex->q_norm_w && !aligned16(ex->q_norm_w)) return false;
    if (ex->sink && !aligned16(ex->sink)) return false;
    if (ex->inv_freq && !aligned16(ex->inv_freq)) return false;
    if (decode && ex->inv_freq && (ex->q_pos == nullptr || !aligned16(ex->q_pos))) return false;
    if (ex->win_len && (!decode || !aligned16(ex->win_len))) return false;
    return ex->norm_eps >= 0.0f;
}

int compress_common(int m, const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride,
                    const float* pos_bias, int32_t B, int64_t n_blocks, hca_kv_layout L,
                    hca_kv_cache out, int64_t entry_begin, const hca_entry_extras* ex, void* stream) {
    REQUIRE(entry_extras_ok(ex));
    REQUIRE(B >= 0 && n_blocks >= 0 && entry_begin >= 0);
    if (!layout_ok(L)) return HCA_ERR_UNSUPPORTED;
    if (B == 0 || n_blocks == 0) return HCA_OK;
    REQ_PTR(x); REQ_PTR(gate); REQ_PTR(pos_bias);
    REQUIRE(cache_ptrs_ok(out));
    REQUIRE(n_blocks * m <= x_seq_stride);
    REQUIRE(entry_begin + n_blocks <= out.capacity);
    return compress_launch(m, x, gate, x_seq_stride, pos_bias, B, n_blocks, L, out, entry_begin, ex,
                           as_stream(stream));
}

}  // namespace

static std::atomic<int> g_launch_budget[3] = {{0}, {0}, {0}};
// a budget set by a library entry for the calls it makes itself (this thread only)
static thread_local int t_budget[3] = {0, 0, 0};
int launch_budget(int op) {
    if (op < 0 || op > 2) return 0;
    return t_budget[op] > 0 ? t_budget[op] : g_launch_budget[op].load();
}
int thread_budget_swap(int op, int max_ctas) {
    if (op < 0 || op > 2) return 0;
    const int prev = t_budget[op];
    t_budget[op] = max_ctas;
    return prev;
}
static std::atomic<int> g_early_query{0};
int early_query() { return g_early_query.load(); }

}  // namespace hca

using namespace hca;

extern "C" {

const char* hca_status_string(int status) {
    switch (status) {
        case HCA_OK: return "ok";
        case HCA_ERR_INVALID_ARG: return "invalid argument";
        case HCA_ERR_UNSUPPORTED: return "unsupported shape or layout";
        case HCA_ERR_CUDA: return "CUDA error";
        case HCA_ERR_WORKSPACE: return "workspace missing or too small";
        case HCA_ERR_SCRATCH_LIMIT: return "request exceeds the library's built-in scratch (16 MiB)";
        default: return "unknown status";
    }
}

int hca_last_cuda_error(void) { return g_last_cuda_error; }


int hca_set_launch_budget(int op, int max_ctas) {
    if ((op != HCA_BUDGET_DENSE_DECODE && op != HCA_BUDGET_SPARSE_DECODE && op != HCA_BUDGET_DECODE_INDEX) ||
        max_ctas < 0)
        return -1;
    return hca::g_launch_budget[op].exchange(max_ctas);
}

int hca_set_early_query(int on) {
    if (on != 0 && on != 1) return -1;
    return hca::g_early_query.exchange(on);
}

int hca_take_device_error(void) {
    const int a = tc_take_device_error(), b = index_take_device_error();
    return (a < 0 || b < 0) ? -1 : (a | b);
}

int csa_compress(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride, const float* pos_bias,
                 int32_t B, int64_t n_blocks, hca_kv_layout layout, hca_kv_cache out,
                 int64_t entry_begin, void* stream) {
    return compress_common(4, x, gate, x_seq_stride, pos_bias, B, n_blocks, layout, out, entry_begin, nullptr,
                           stream);
}

int csa_compress_ex(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride, const float* pos_bias,
                    int32_t B, int64_t n_blocks, hca_kv_layout layout, hca_kv_cache out,
                    int64_t entry_begin, const hca_entry_extras* ex, void* stream) {
    return compress_common(4, x, gate, x_seq_stride, pos_bias, B, n_blocks, layout, out, entry_begin, ex, stream);
}

int hca_compress_ex(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride, const float* pos_bias,
                    int32_t B, int64_t n_blocks, hca_kv_layout layout, hca_kv_cache out,
                    int64_t entry_begin, const hca_entry_extras* ex, void* stream) {
    return compress_common(128, x, gate, x_seq_stride, pos_bias, B, n_blocks, layout, out, entry_begin, ex,
                           stream);
}

int kv_token_prep(const uint16_t* x, const int32_t* pos, int64_t n, hca_kv_layout layout,
                  const hca_entry_extras* ex, uint16_t* out, void* stream) {
    REQUIRE(n >= 0);
    if (!layout_ok(layout)) return HCA_ERR_UNSUPPORTED;
    if (n == 0) return HCA_OK;
    REQ_PTR(x); REQ_PTR(pos); REQ_PTR(out);
    REQUIRE(entry_extras_ok(ex));
    return token_prep_launch(x, pos, n, layout, ex, out, as_stream(stream));
}

int hca_compress(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride, const float* pos_bias,
                 int32_t B, int64_t n_blocks, hca_kv_layout layout, hca_kv_cache out,
                 int64_t entry_begin, void* stream) {
    return compress_common(128, x, gate, x_seq_stride, pos_bias, B, n_blocks, layout, out, entry_begin, nullptr,
                           stream);
}

static bool heads_ok(int Hi, int c) { return (Hi >= 1 && Hi <= 8) || (Hi == 64 && c == 128); }

int lightning_index_ex(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                       const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                       int32_t B, int32_t Tq, int64_t Nc_cap, int32_t Hi, int32_t c, int32_t m,
                       int32_t score_bf16, void* scores, void* stream) {
    REQUIRE(B >= 0 && Tq >= 0 && Nc_cap >= 0 && m >= 1);
    if (c != 64 && c != 128) return HCA_ERR_UNSUPPORTED;
    if (!heads_ok(Hi, c)) return HCA_ERR_UNSUPPORTED;
    if (score_bf16 && !(c == 128 && (Hi == 4 || Hi == 64))) return HCA_ERR_UNSUPPORTED;
    if (B == 0 || Tq == 0 || Nc_cap == 0) return HCA_OK;
    REQ_PTR(q_codes); REQ_PTR(q_sf); REQ_PTR(w); REQ_PTR(k_codes); REQ_PTR(k_sf); REQ_PTR(q_pos); REQ_PTR(scores);
    return index_launch(q_codes, q_sf, w, k_codes, k_sf, q_pos, B, Tq, Nc_cap, Hi, c, m, scores, as_stream(stream),
                        score_bf16 != 0);
}

int lightning_index(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                    const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                    int32_t B, int32_t Tq, int64_t Nc_cap, int32_t Hi, int32_t c, int32_t m,
                    float* scores, void* stream) {
    return lightning_index_ex(q_codes, q_sf, w, k_codes, k_sf, q_pos, B, Tq, Nc_cap, Hi, c, m, 0, scores, stream);
}

size_t topk_select_workspace_size(int32_t R, int64_t Nc_cap, int32_t k) {
    (void)k;
    if (R <= 0 || Nc_cap <= 0 || !topk_wide_preferred(R, Nc_cap)) return 0;
    return topk_wide_ws_bytes(R, Nc_cap);
}

size_t topk_select_ex_workspace_size(int32_t R, int64_t Nc_cap, int32_t k, int32_t score_bf16) {
    if (!score_bf16) return topk_select_workspace_size(R, Nc_cap, k);
    if (R <= 0 || Nc_cap <= 0) return 0;
    return topk_wide_ws_bytes(R, Nc_cap);
}

int topk_select(const float* scores, const int32_t* q_pos, int32_t R, int64_t Nc_cap, int32_t m, int32_t k,
                int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, void* stream) {
    REQUIRE(R >= 0 && Nc_cap >= 0 && m >= 1);
    if (k < 1 || k > 4096) return HCA_ERR_UNSUPPORTED;
    if (R == 0) return HCA_OK;
    REQ_PTR(q_pos); REQ_PTR(idx); REQ_PTR(count);
    if (Nc_cap > 0) REQ_PTR(scores);
    if (Nc_cap > 16 * 32768LL && ws_bytes < topk_select_workspace_size(R, Nc_cap, k)) return HCA_ERR_WORKSPACE;
    return topk_launch(scores, q_pos, R, Nc_cap, m, k, idx, count, ws, ws_bytes, as_stream(stream));
}

int topk_select_ex(const void* scores, int32_t score_bf16, const int32_t* q_pos, int32_t R, int64_t Nc_cap,
                   int32_t m, int32_t k, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, void* stream) {
    if (!score_bf16)
        return topk_select(static_cast<const float*>(scores), q_pos, R, Nc_cap, m, k, idx, count, ws, ws_bytes,
                           stream);
    REQUIRE(R >= 0 && Nc_cap >= 0 && m >= 1);
    if (k < 1 || k > 4096) return HCA_ERR_UNSUPPORTED;
    if (R == 0) return HCA_OK;
    REQ_PTR(q_pos); REQ_PTR(idx); REQ_PTR(count); REQ_PTR(scores);
    REQUIRE(Nc_cap >= 1);
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) ||
        ws_bytes < topk_select_ex_workspace_size(R, Nc_cap, k, 1))
        return HCA_ERR_WORKSPACE;
    if (R > 65535 || Nc_cap > 0x7FFFFFFFLL) return HCA_ERR_UNSUPPORTED;
    return topk_wide_launch(scores, q_pos, R, Nc_cap, m, k, idx, count, ws, as_stream(stream), true);
}

static int record_event(void* ev, cudaStream_t st) {
    if (ev == nullptr) return HCA_OK;
    const cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(ev), st);
    if (e != cudaSuccess) { hca::set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    return HCA_OK;
}

size_t lightning_index_topk_workspace_size(int32_t B, int64_t Nc_cap, int32_t k) {
    return topk_select_workspace_size(B, Nc_cap, k);
}

size_t lightning_index_topk_ex_workspace_size(int32_t B, int64_t Nc_cap, int32_t k, int32_t score_bf16) {
    return topk_select_ex_workspace_size(B, Nc_cap, k, score_bf16);
}

int lightning_index_topk_ex(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                            const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                            int32_t B, int64_t Nc_cap, int32_t Hi, int32_t c, int32_t m, int32_t k,
                            int32_t score_bf16, void* scores, int32_t* idx, int32_t* count, void* ws,
                            size_t ws_bytes, void* index_done, void* stream) {
    REQUIRE(B >= 0 && Nc_cap >= 0 && m >= 1);
    if (c != 64 && c != 128) return HCA_ERR_UNSUPPORTED;
    if (!heads_ok(Hi, c)) return HCA_ERR_UNSUPPORTED;
    if (k < 1 || k > 4096) return HCA_ERR_UNSUPPORTED;
    if (score_bf16 && !(c == 128 && (Hi == 4 || Hi == 64))) return HCA_ERR_UNSUPPORTED;
    if (B == 0) return HCA_OK;
    REQ_PTR(q_pos); REQ_PTR(idx); REQ_PTR(count);
    if (score_bf16) REQUIRE(Nc_cap >= 1);
    if (Nc_cap > 0) { REQ_PTR(q_codes); REQ_PTR(q_sf); REQ_PTR(w); REQ_PTR(k_codes); REQ_PTR(k_sf); REQ_PTR(scores); }
    const size_t need = topk_select_ex_workspace_size(B, Nc_cap, k, score_bf16);
    if ((Nc_cap > 16 * 32768LL || score_bf16) && ws_bytes < need) return HCA_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    if (need > 0 && ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0) {
        // fused: the indexer also builds each row's key histogram
        int rc = topk_wide_clear(ws, B, Nc_cap, st);
        if (rc != HCA_OK) return rc;
        int64_t stride = 0;
        uint32_t* hist = topk_wide_hist(ws, Nc_cap, &stride);
        rc = index_launch_hist(q_codes, q_sf, w, k_codes, k_sf, q_pos, B, Nc_cap, Hi, c, m, scores, hist, stride, st,
                               score_bf16 != 0);
        if (rc == HCA_OK) {
            rc = record_event(index_done, st);
            if (rc != HCA_OK) return rc;
            return topk_wide_select(scores, q_pos, B, Nc_cap, m, k, idx, count, ws, st, score_bf16 != 0);
        }
        if (rc != HCA_ERR_UNSUPPORTED) return rc;
    }
    // separate calls
    if (Nc_cap > 0) {
        const int rc = index_launch(q_codes, q_sf, w, k_codes, k_sf, q_pos, B, 1, Nc_cap, Hi, c, m, scores, st,
                                    score_bf16 != 0);
        if (rc != HCA_OK) return rc;
    }
    const int rc = record_event(index_done, st);
    if (rc != HCA_OK) return rc;
    if (score_bf16) {
        if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return HCA_ERR_WORKSPACE;
        return topk_wide_launch(scores, q_pos, B, Nc_cap, m, k, idx, count, ws, st, true);
    }
    return topk_launch(static_cast<const float*>(scores), q_pos, B, Nc_cap, m, k, idx, count, ws, ws_bytes, st);
}

int lightning_index_topk(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                         const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                         int32_t B, int64_t Nc_cap, int32_t Hi, int32_t c, int32_t m, int32_t k,
                         float* scores, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                         void* index_done, void* stream) {
    return lightning_index_topk_ex(q_codes, q_sf, w, k_codes, k_sf, q_pos, B, Nc_cap, Hi, c, m, k, 0, scores, idx,
                                   count, ws, ws_bytes, index_done, stream);
}

size_t compressed_attn_decode_workspace_size(int32_t B, int32_t H, hca_kv_layout layout, int32_t max_comp, int32_t W) {
    if (B <= 0 || max_comp < 0 || W < 0 || !layout_ok(layout)) return 0;
    return decode_ws_bytes(B, H, layout.d, max_comp, W);
}

int compressed_attn_decode_ex(const uint16_t* q, int32_t B, int32_t H, hca_kv_layout layout, hca_kv_cache kv,
                              const int32_t* idx, int32_t idx_stride, const int32_t* n_comp, int32_t max_comp,
                              const uint16_t* window, int32_t W, float softmax_scale, const hca_attn_extras* ex,
                              uint16_t* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
    REQUIRE(B >= 0 && max_comp >= 0 && W >= 0);
    if (!layout_ok(layout)) return HCA_ERR_UNSUPPORTED;
    if (!((layout.d == 512 && H == 64) || (layout.d == 128 && (H == 64 || (H >= 1 && H <= 16)))))
        return HCA_ERR_UNSUPPORTED;
    if (W > 4096) return HCA_ERR_UNSUPPORTED;
    if (B == 0) return HCA_OK;
    REQ_PTR(q); REQ_PTR(n_comp); REQ_PTR(out);
    REQUIRE(cache_ptrs_ok(kv));
    if (W > 0) REQ_PTR(window);
    if (idx) { REQUIRE(aligned16(idx) && idx_stride >= max_comp); }
    if (lse) REQUIRE(aligned16(lse));
    if (ws) REQUIRE(aligned16(ws));
    REQUIRE(attn_extras_ok(ex, true));
    return attn_decode_launch(q, B, H, layout, kv, idx, idx_stride, n_comp, max_comp, window, W, softmax_scale,
                              ex, out, lse, ws, ws_bytes, as_stream(stream));
}

int compressed_attn_decode(const uint16_t* q, int32_t B, int32_t H, hca_kv_layout layout, hca_kv_cache kv,
                           const int32_t* idx, int32_t idx_stride, const int32_t* n_comp, int32_t max_comp,
                           const uint16_t* window, int32_t W, float softmax_scale, uint16_t* out, float* lse,
                           void* ws, size_t ws_bytes, void* stream) {
    return compressed_attn_decode_ex(q, B, H, layout, kv, idx, idx_stride, n_comp, max_comp, window, W,
                                     softmax_scale, nullptr, out, lse, ws, ws_bytes, stream);
}

int kv_state_append(const uint16_t* x, const uint16_t* gate, const uint16_t* win_x, int32_t B, int32_t d,
                    int64_t pos, uint16_t* window, int32_t W, uint16_t* tail_x, uint16_t* tail_gate,
                    int32_t m, void* stream) {
    REQUIRE(B >= 0 && pos >= 0 && W >= 0 && m >= 0 && d > 0 && d % 8 == 0);
    if (B == 0) return HCA_OK;
    REQ_PTR(x);
    if (W > 0) REQ_PTR(window);
    if (win_x) REQ_PTR(win_x);
    if (m > 0 && tail_x) { REQ_PTR(tail_x); REQ_PTR(gate); REQ_PTR(tail_gate); }
    return state_append_launch(x, gate, win_x, B, d, pos, window, W, tail_x, tail_gate, m, as_stream(stream));
}

int csa_compress_overlap(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                         const uint16_t* a_prev, const uint16_t* za_prev, int64_t x_seq_stride,
                         const float* pos_bias, int32_t B, int64_t n_blocks, hca_kv_layout layout,
                         hca_kv_cache out, int64_t entry_begin, void* stream) {
    REQUIRE(B >= 0 && n_blocks >= 0 && entry_begin >= 0);
    if (!layout_ok(layout)) return HCA_ERR_UNSUPPORTED;
    if (B == 0 || n_blocks == 0) return HCA_OK;
    REQ_PTR(xa); REQ_PTR(za); REQ_PTR(xb); REQ_PTR(zb); REQ_PTR(pos_bias);
    REQUIRE((a_prev == nullptr) == (za_prev == nullptr));
    if (a_prev) { REQ_PTR(a_prev); REQ_PTR(za_prev); }
    REQUIRE(cache_ptrs_ok(out));
    REQUIRE(n_blocks * 4 <= x_seq_stride);
    REQUIRE(entry_begin + n_blocks <= out.capacity);
    return overlap_launch(xa, za, xb, zb, a_prev, za_prev, x_seq_stride, pos_bias, B, n_blocks, layout.d,
                          layout.d_rope, layout.scale_group, out.codes, out.scales, out.rope, nullptr, out.capacity,
                          entry_begin, false, as_stream(stream));
}

int indexer_key_compress(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                         const uint16_t* a_prev, const uint16_t* za_prev, int64_t x_seq_stride,
                         const float* pos_bias, int32_t B, int64_t n_blocks, int32_t c,
                         uint8_t* k_codes, uint8_t* k_sf, int64_t capacity, int64_t entry_begin, void* stream) {
    REQUIRE(B >= 0 && n_blocks >= 0 && entry_begin >= 0 && capacity >= 0);
    if (c != 64 && c != 128) return HCA_ERR_UNSUPPORTED;
    if (B == 0 || n_blocks == 0) return HCA_OK;
    REQ_PTR(xa); REQ_PTR(za); REQ_PTR(xb); REQ_PTR(zb); REQ_PTR(pos_bias); REQ_PTR(k_codes); REQ_PTR(k_sf);
    REQUIRE((a_prev == nullptr) == (za_prev == nullptr));
    if (a_prev) { REQ_PTR(a_prev); REQ_PTR(za_prev); }
    REQUIRE(n_blocks * 4 <= x_seq_stride);
    REQUIRE(entry_begin + n_blocks <= capacity);
    return overlap_launch(xa, za, xb, zb, a_prev, za_prev, x_seq_stride, pos_bias, B, n_blocks, c, 0, 32, k_codes,
                          nullptr, nullptr, k_sf, capacity, entry_begin, true, as_stream(stream));
}

int compressed_attn_prefill_ex(const uint16_t* q, int32_t Tq, int32_t H, int32_t p0, int32_t m,
                               hca_kv_layout layout, hca_kv_cache kv, const int32_t* idx, int32_t idx_stride,
                               const int32_t* count, const uint16_t* raw, int32_t W, float softmax_scale,
                               const hca_attn_extras* ex, uint16_t* out, void* stream) {
    REQUIRE(Tq >= 0 && p0 >= 0 && W >= 1);
    if (!layout_ok(layout)) return HCA_ERR_UNSUPPORTED;
    if (!((layout.d == 512 && H == 64) || (layout.d == 128 && (H == 64 || (H >= 1 && H <= 16)))))
        return HCA_ERR_UNSUPPORTED;
    if (W > 4096) return HCA_ERR_UNSUPPORTED;
    if (Tq == 0) return HCA_OK;
    REQ_PTR(q); REQ_PTR(out); REQ_PTR(raw);
    REQUIRE(cache_ptrs_ok(kv));
    if (idx) { REQUIRE(aligned16(idx) && count != nullptr && aligned16(count) && idx_stride >= 0); }
    else { REQUIRE(m >= 1); }
    REQUIRE(attn_extras_ok(ex, false));
    return attn_prefill_launch(q, Tq, H, p0, m, layout, kv, idx, idx_stride, count, raw, W, softmax_scale, ex, out,
                               as_stream(stream));
}

int compressed_attn_prefill(const uint16_t* q, int32_t Tq, int32_t H, int32_t p0, int32_t m,
                            hca_kv_layout layout, hca_kv_cache kv, const int32_t* idx, int32_t idx_stride,
                            const int32_t* count, const uint16_t* raw, int32_t W, float softmax_scale,
                            uint16_t* out, void* stream) {
    return compressed_attn_prefill_ex(q, Tq, H, p0, m, layout, kv, idx, idx_stride, count, raw, W, softmax_scale,
                                      nullptr, out, stream);
}

}  // extern "C"
