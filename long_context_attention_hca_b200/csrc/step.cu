// step.cu -- one decode step of a CSA layer and an HCA layer from host
// memory to host memory through the library alone: the query copies in, the
// fused index + top-k, both attention calls and the output copies out, on two
// streams ("DeepSeek V4 ..." note, sections 7 and 8: the CSA path -- indexer,
// top-k, attention over the selected entries and the window -- and the HCA
// path -- dense attention over every entry and the window -- of one decode
// position).
//
// Schedule (the two paths share no data):
//   side:   waits ev_fork | H2D indexer query (records ev_iq) | index + top-k
//           (records ev_index) | waits ev_q | CSA attention | D2H CSA output
//           (records ev_join)
//   stream: records ev_fork | waits ev_iq | H2D CSA query (records ev_q) |
//           H2D HCA query | waits ev_index | HCA attention | D2H HCA output |
//           waits ev_join
// The CSA chain is the critical path, so the side stream should have the
// higher priority; the HCA launch waits for the indexer, which fills every SM
// anyway.  The indexer query (a few hundred bytes) crosses alone: queued
// beside the attention queries it would share the link with them and the
// indexer would start late; those cross while the indexer runs.  Every copy
// is one cudaMemcpyAsync.  When the caller states it (plan->packed), the
// indexer query's three arrays take one copy, and the two outputs take one,
// on `stream` after the join (one copy of 512 KB costs about 12.7 us on a
// PCIe link, two of 256 KB about 8 us each).  Adjacent pointers alone do not
// prove one allocation, and a copy across two pinned allocations is refused,
// hence the flag.  The host buffers should be pinned so that the copies are
// asynchronous.
#include "common.cuh"

using namespace hca;

namespace {
int rec(void* ev, void* st) {
    const cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(ev), as_stream(st));
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    return HCA_OK;
}
int wait(void* st, void* ev) {
    const cudaError_t e = cudaStreamWaitEvent(as_stream(st), static_cast<cudaEvent_t>(ev), 0);
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    return HCA_OK;
}
int cpy(void* dst, const void* src, size_t n, cudaMemcpyKind kind, void* st) {
    if (n == 0) return HCA_OK;
    const cudaError_t e = cudaMemcpyAsync(dst, src, n, kind, as_stream(st));
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    return HCA_OK;
}
}  // namespace

#define HCA_TRY(x) do { const int _rc = (x); if (_rc != HCA_OK) return _rc; } while (0)

extern "C" int hca_decode_step_host(const hca_decode_step_plan* p, const uint16_t* h_q_csa, const uint16_t* h_q_hca,
                                    const uint8_t* h_iq_codes, const uint8_t* h_iq_sf, const float* h_iq_w,
                                    uint16_t* h_out_csa, uint16_t* h_out_hca, void* stream) {
    if (!p || !h_q_csa || !h_q_hca || !h_iq_codes || !h_iq_sf || !h_iq_w || !h_out_csa || !h_out_hca)
        return HCA_ERR_INVALID_ARG;
    if (!p->side_stream || !p->ev_fork || !p->ev_index || !p->ev_q || !p->ev_join || !p->ev_iq)
        return HCA_ERR_INVALID_ARG;
    if (p->B <= 0 || p->H <= 0 || p->Hi <= 0 || p->c <= 0 || p->layout.d <= 0 || p->hca_ctas < 0)
        return HCA_ERR_INVALID_ARG;
    const size_t d = static_cast<size_t>(p->layout.d);
    const size_t q_bytes = static_cast<size_t>(p->B) * p->H * d * 2;
    const size_t iqc = static_cast<size_t>(p->B) * p->Hi * (p->c / 2);
    const size_t iqs = static_cast<size_t>(p->B) * p->Hi * (p->c / 32);
    const size_t iqw = static_cast<size_t>(p->B) * p->Hi * sizeof(float);
    if (p->packed & ~3) return HCA_ERR_INVALID_ARG;
    // packed indexer query: scales and weights follow the codes, each from the next
    // 16-byte boundary, in host and in device memory
    const uint8_t* hc = h_iq_codes;
    const uint8_t* dc = p->iq_codes;
    const size_t o_sf = (iqc + 15) & ~static_cast<size_t>(15), o_w = o_sf + ((iqs + 15) & ~static_cast<size_t>(15));
    const bool iq_packed = (p->packed & 1) != 0;
    if (iq_packed && !(reinterpret_cast<const uint8_t*>(h_iq_sf) == hc + o_sf &&
                       reinterpret_cast<const uint8_t*>(h_iq_w) == hc + o_w &&
                       reinterpret_cast<const uint8_t*>(p->iq_sf) == dc + o_sf &&
                       reinterpret_cast<const uint8_t*>(p->iq_w) == dc + o_w))
        return HCA_ERR_INVALID_ARG;
    // packed outputs: both back to back (either order) in device and in host memory
    // alike, one copy of both once the two paths have joined
    const size_t n_out = q_bytes / 2;
    const uint16_t* d_first = nullptr;
    uint16_t* h_first = nullptr;
    if (p->packed & 2) {
        if (p->out_hca == p->out_csa + n_out && h_out_hca == h_out_csa + n_out) {
            d_first = p->out_csa; h_first = h_out_csa;
        } else if (p->out_csa == p->out_hca + n_out && h_out_csa == h_out_hca + n_out) {
            d_first = p->out_hca; h_first = h_out_hca;
        } else {
            return HCA_ERR_INVALID_ARG;
        }
    }
    void* side = p->side_stream;
    HCA_TRY(rec(p->ev_fork, stream));
    HCA_TRY(wait(side, p->ev_fork));
    // CSA chain on the side stream: the indexer query (a few hundred bytes), then
    // index + top-k, attention and the output
    if (iq_packed) {
        HCA_TRY(cpy(p->iq_codes, h_iq_codes, o_w + iqw, cudaMemcpyHostToDevice, side));
    } else {
        HCA_TRY(cpy(p->iq_codes, h_iq_codes, iqc, cudaMemcpyHostToDevice, side));
        HCA_TRY(cpy(p->iq_sf, h_iq_sf, iqs, cudaMemcpyHostToDevice, side));
        HCA_TRY(cpy(p->iq_w, h_iq_w, iqw, cudaMemcpyHostToDevice, side));
    }
    HCA_TRY(rec(p->ev_iq, side));
    HCA_TRY(lightning_index_topk(p->iq_codes, p->iq_sf, p->iq_w, p->k_codes, p->k_sf, p->q_pos, p->B,
                                 p->csa_entries, p->Hi, p->c, 4, p->k, p->scores, p->idx, p->count, p->topk_ws,
                                 p->topk_ws_bytes, p->ev_index, side));
    // the attention queries cross while the indexer runs
    HCA_TRY(wait(stream, p->ev_iq));
    HCA_TRY(cpy(p->q_csa, h_q_csa, q_bytes, cudaMemcpyHostToDevice, stream));
    HCA_TRY(rec(p->ev_q, stream));
    HCA_TRY(cpy(p->q_hca, h_q_hca, q_bytes, cudaMemcpyHostToDevice, stream));
    // CSA attention over the selected entries and the window, then its output
    HCA_TRY(wait(side, p->ev_q));
    const int32_t kmax = static_cast<int32_t>(p->csa_entries < p->k ? p->csa_entries : p->k);
    HCA_TRY(compressed_attn_decode(p->q_csa, p->B, p->H, p->layout, p->csa_cache, p->idx, p->k, p->count, kmax,
                                   p->csa_window, p->W, p->softmax_scale, p->out_csa, nullptr, p->ws_csa,
                                   p->ws_csa_bytes, side));
    if (!d_first) HCA_TRY(cpy(h_out_csa, p->out_csa, q_bytes, cudaMemcpyDeviceToHost, side));
    HCA_TRY(rec(p->ev_join, side));
    // HCA: dense attention once the indexer has run, on at most hca_ctas CTAs (by
    // default the SMs that the select's CTAs leave, at least half) so that the CSA
    // chain's select and attention keep the rest; then its output
    HCA_TRY(wait(stream, p->ev_index));
    const int prev = thread_budget_swap(HCA_BUDGET_DENSE_DECODE, p->hca_ctas > 0 ? p->hca_ctas : dense_beside_select(p->B));
    const int rc = compressed_attn_decode(p->q_hca, p->B, p->H, p->layout, p->hca_cache, nullptr, 0, p->hca_n,
                                          p->hca_max, p->hca_window, p->W, p->softmax_scale, p->out_hca, nullptr,
                                          p->ws_hca, p->ws_hca_bytes, stream);
    thread_budget_swap(HCA_BUDGET_DENSE_DECODE, prev);
    HCA_TRY(rc);
    if (!d_first) HCA_TRY(cpy(h_out_hca, p->out_hca, q_bytes, cudaMemcpyDeviceToHost, stream));
    HCA_TRY(wait(stream, p->ev_join));
    if (d_first) HCA_TRY(cpy(h_first, d_first, 2 * q_bytes, cudaMemcpyDeviceToHost, stream));
    return HCA_OK;
}
