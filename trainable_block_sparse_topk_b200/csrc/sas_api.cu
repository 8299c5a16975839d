// sas_api.cu -- the C ABI of libsas (declared in include/sas.h).
//
// Every entry point validates its arguments completely before it launches
// anything, carves its workspace from the caller's buffer, and enqueues its
// kernels on the caller's stream. Nothing here allocates, frees or
// synchronises the host.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace sas {

// Readers for the wait-timeout counters of the translation units that wait.
cudaError_t read_decode_timeouts(unsigned int* out);
cudaError_t read_bwd_tc_timeouts(unsigned int* out);
cudaError_t read_fwd_rows_timeouts(unsigned int* out);
cudaError_t set_decode_wait_limit(unsigned long long ns);
cudaError_t set_bwd_tc_wait_limit(unsigned long long ns);
cudaError_t set_fwd_rows_wait_limit(unsigned long long ns);

static std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// ------------------------------------------------------- per-kernel timing ---
namespace {
struct TimingRec {
    const char* name;
    cudaEvent_t a, b;
};
std::mutex g_tmu;
std::atomic<bool> g_timing{false};
std::atomic<bool> g_timing_err{false};
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_pool;
std::string g_filter;   // ",a,b," or "*"

bool timed(const char* name) {   // g_tmu held
    if (g_filter == "*") return true;
    return g_filter.find("," + std::string(name) + ",") != std::string::npos;
}

cudaEvent_t take_event() {   // g_tmu held
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}
}  // namespace

KernelTimer::KernelTimer(const char* name, cudaStream_t st) : name_(name), st_(st), start_(nullptr) {
    if (!g_timing.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_tmu);
    if (!timed(name)) return;
    cudaEvent_t e = take_event();
    if (e == nullptr || cudaEventRecord(e, st_) != cudaSuccess) {
        g_timing_err = true;
        if (e) g_pool.push_back(e);
        return;
    }
    start_ = e;
}

KernelTimer::~KernelTimer() {
    if (start_ == nullptr) return;
    std::lock_guard<std::mutex> lk(g_tmu);
    cudaEvent_t a = static_cast<cudaEvent_t>(start_);
    cudaEvent_t b = take_event();
    if (b == nullptr || cudaEventRecord(b, st_) != cudaSuccess) {
        g_timing_err = true;
        g_pool.push_back(a);
        if (b) g_pool.push_back(b);
        return;
    }
    g_recs.push_back({name_, a, b});
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

enum class Kind { kTopk, kTrain, kDecode };

sas_status make_shape(const sas_desc* d, Kind kind, Shape* s) {
    if (!d || !s) return SAS_ERR_INVALID_ARG;
    if (d->batch < 1 || d->seq_len < 1 || d->q_offset < 0 || d->n_q_heads < 1 || d->n_kv_heads < 1 ||
        d->head_dim < 1 || d->block_size < 1 || d->top_k < 1)
        return SAS_ERR_INVALID_ARG;
    if (d->n_q_heads % d->n_kv_heads != 0) return SAS_ERR_INVALID_ARG;
    if (d->dtype != SAS_DT_BF16 && d->dtype != SAS_DT_FP32) return SAS_ERR_INVALID_ARG;
    if (d->gate < SAS_GATE_SOFTMAX || d->gate > SAS_GATE_STE) return SAS_ERR_INVALID_ARG;
    if (d->select_heads != 0 && d->select_heads != 1) return SAS_ERR_INVALID_ARG;
    if (!(d->softmax_scale <= 0.f) && !std::isfinite(d->softmax_scale)) return SAS_ERR_INVALID_ARG;
    if (std::isnan(d->softmax_scale)) return SAS_ERR_INVALID_ARG;
    const int G = d->n_q_heads / d->n_kv_heads;
    if (G > 8) return SAS_ERR_UNSUPPORTED;
    if (d->head_dim != 64 && d->head_dim != 128) return SAS_ERR_UNSUPPORTED;
    if (d->block_size != 32 && d->block_size != 64) return SAS_ERR_UNSUPPORTED;
    if (d->top_k > 64) return SAS_ERR_UNSUPPORTED;
    const int64_t len = (int64_t)d->q_offset + d->seq_len;
    if (len > (int64_t)1 << 30) return SAS_ERR_UNSUPPORTED;
    if (!topk_row_supported((len - 1) / d->block_size)) return SAS_ERR_UNSUPPORTED;
    if (kind == Kind::kTrain) {
        if (d->q_offset != 0 || d->seq_len % d->block_size != 0) return SAS_ERR_UNSUPPORTED;
    }
    if (kind == Kind::kDecode && d->seq_len != 1) return SAS_ERR_INVALID_ARG;
    s->B = d->batch;
    s->T = d->seq_len;
    s->q_offset = d->q_offset;
    s->Hq = d->n_q_heads;
    if (d->select_heads) {          // one selection group per query head
        s->Hkv = d->n_q_heads;
        s->G = 1;
        s->Hkvp = d->n_kv_heads;
        s->kvdiv = G;
    } else {
        s->Hkv = d->n_kv_heads;
        s->G = G;
        s->Hkvp = d->n_kv_heads;
        s->kvdiv = 1;
    }
    s->D = d->head_dim;
    s->bs = d->block_size;
    s->K = d->top_k;
    s->NB = (int)((len + d->block_size - 1) / d->block_size);
    s->nT = d->seq_len / d->block_size;
    s->scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.f / std::sqrt((float)d->head_dim);
    s->dtype = d->dtype;
    s->gate = d->gate;
    if ((int64_t)s->B * s->Hkv * s->T > ((int64_t)1 << 31) / 64) return SAS_ERR_UNSUPPORTED;
    return SAS_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Training workspace layout (each piece 256-byte aligned).
struct TrainWs {
    size_t maskT, Dd, gsum, dq_acc, dkv32, stream, flag, total;
};

TrainWs bwd_layout(const Shape& s) {
    TrainWs w{};
    size_t off = 0;
    w.maskT = off; off += align256(sizeof(uint64_t) * (size_t)s.B * s.Hkv * s.NB * s.nT);
    w.Dd = off;    off += align256(sizeof(float) * (size_t)s.B * s.Hq * s.T);
    w.gsum = off;  off += align256(sizeof(float) * (size_t)s.B * s.Hkv * s.T * s.K);
    w.dq_acc = off;
    if (s.dtype != SAS_DT_FP32) off += align256(sizeof(float) * (size_t)s.B * s.Hq * s.T * s.D);
    w.dkv32 = off;    // per-query-head selection: fp32 dK, dV per selection group
    if (s.kvdiv > 1) off += 2 * align256(sizeof(float) * (size_t)s.B * s.Hkv * s.T * s.D);
    w.stream = off;   // the tensor-core backward's per-block token streams
    if (bwd_tc_supported(s)) off += align256(bwd_tc_ws_bytes(s));
    w.flag = off;     // set by a CTA that gave up on a wait
    off += 256;
    w.total = off;
    return w;
}

// Forward workspace: column bitmap, then the gathered-row kernels' row
// statistics and fp32 output accumulator.
size_t fwd_ws_bytes(const Shape& s) {
    if (!fwd_rows_supported(s)) return 0;
    return align256(sizeof(uint64_t) * (size_t)s.B * s.Hkv * s.NB * s.nT) + align256(fwd_rows_ws_bytes(s));
}

size_t ws_bytes(int op, const Shape& s) {
    switch (op) {
        case SAS_OP_TOPK: return 0;
        case SAS_OP_FWD: return fwd_ws_bytes(s);
        case SAS_OP_BWD: return bwd_layout(s).total;
        case SAS_OP_DECODE: return align256(decode_ws_bytes(s));
        default: return 0;
    }
}

sas_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SAS_OK : SAS_ERR_CUDA; }

template <typename... P>
bool any_null(P... p) { return ((p == nullptr) || ...); }
template <typename... P>
bool any_misaligned(P... p) { return (!aligned16(p) || ...); }

}  // namespace

sas_status check_decode_args(const sas_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                             int64_t cache_stride_tokens, const int32_t* idx, const float* gate_logit,
                             const int32_t* n_sel, const void* o, Shape* s) {
    sas_status st = make_shape(desc, Kind::kDecode, s);
    if (st != SAS_OK) return st;
    if (any_null(q, k_cache, v_cache, o)) return SAS_ERR_INVALID_ARG;
    if (idx != nullptr && any_null(gate_logit, n_sel)) return SAS_ERR_INVALID_ARG;
    if (cache_stride_tokens < (int64_t)s->q_offset + 1) return SAS_ERR_INVALID_ARG;
    if (any_misaligned(q, k_cache, v_cache, o)) return SAS_ERR_MISALIGNED;
    if (idx != nullptr && any_misaligned(idx, gate_logit, n_sel)) return SAS_ERR_MISALIGNED;
    return SAS_OK;
}

}  // namespace sas

using namespace sas;

extern "C" {

const char* sas_status_string(sas_status st) {
    switch (st) {
        case SAS_OK: return "ok";
        case SAS_ERR_INVALID_ARG: return "invalid argument";
        case SAS_ERR_UNSUPPORTED: return "unsupported shape or option";
        case SAS_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case SAS_ERR_WORKSPACE: return "workspace missing or too small";
        case SAS_ERR_CUDA: return "CUDA launch or runtime error";
        default: return "unknown status";
    }
}

sas_status sas_workspace_size(int32_t op, const sas_desc* desc, size_t* bytes) {
    if (!bytes) return SAS_ERR_INVALID_ARG;
    if (op < SAS_OP_TOPK || op > SAS_OP_DECODE) return SAS_ERR_INVALID_ARG;
    const Kind kind = op == SAS_OP_TOPK ? Kind::kTopk : (op == SAS_OP_DECODE ? Kind::kDecode : Kind::kTrain);
    Shape s;
    sas_status st = make_shape(desc, kind, &s);
    if (st != SAS_OK) return st;
    *bytes = ws_bytes(op, s);
    return SAS_OK;
}

sas_status sas_block_topk(const sas_desc* desc, const float* scores, int32_t* idx, float* gate_logit,
                          float* score_lse, int32_t* n_sel, void* stream) {
    Shape s;
    sas_status st = make_shape(desc, Kind::kTopk, &s);
    if (st != SAS_OK) return st;
    if (any_null(scores, idx, gate_logit, score_lse, n_sel)) return SAS_ERR_INVALID_ARG;
    if (any_misaligned(scores, idx, gate_logit, score_lse, n_sel)) return SAS_ERR_MISALIGNED;
    return cuda_status(launch_block_topk(s, scores, nullptr, idx, gate_logit, score_lse, n_sel, (cudaStream_t)stream));
}

sas_status sas_block_topk_varlen(const sas_desc* desc, const float* scores, const int32_t* seq_lens, int32_t* idx,
                                 float* gate_logit, float* score_lse, int32_t* n_sel, void* stream) {
    Shape s;
    sas_status st = make_shape(desc, Kind::kDecode, &s);
    if (st != SAS_OK) return st;
    if (any_null(scores, seq_lens, idx, gate_logit, score_lse, n_sel)) return SAS_ERR_INVALID_ARG;
    if (any_misaligned(scores, seq_lens, idx, gate_logit, score_lse, n_sel)) return SAS_ERR_MISALIGNED;
    return cuda_status(launch_block_topk(s, scores, seq_lens, idx, gate_logit, score_lse, n_sel,
                                         (cudaStream_t)stream));
}

sas_status sas_gated_attn_fwd(const sas_desc* desc, const void* q, const void* k, const void* v,
                              const int32_t* idx, const float* gate_logit, const int32_t* n_sel, void* o,
                              float* attn_lse, void* ws, size_t ws_bytes_, void* stream) {
    Shape s;
    sas_status st = make_shape(desc, Kind::kTrain, &s);
    if (st != SAS_OK) return st;
    if (any_null(q, k, v, idx, gate_logit, n_sel, o, attn_lse)) return SAS_ERR_INVALID_ARG;
    if (any_misaligned(q, k, v, idx, gate_logit, n_sel, o, attn_lse)) return SAS_ERR_MISALIGNED;
    const size_t need = ws_bytes(SAS_OP_FWD, s);
    if (need > 0 && (ws == nullptr || ws_bytes_ < need)) return SAS_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return SAS_ERR_MISALIGNED;
    cudaStream_t cs = (cudaStream_t)stream;
    if (fwd_rows_supported(s)) {
        unsigned char* w = static_cast<unsigned char*>(ws);
        uint64_t* maskT = reinterpret_cast<uint64_t*>(w);
        void* rows_ws = w + align256(sizeof(uint64_t) * (size_t)s.B * s.Hkv * s.NB * s.nT);
        cudaError_t e = launch_sel_bitmap_T(s, idx, n_sel, maskT, cs);
        if (e == cudaSuccess) e = launch_fwd_rows(s, q, k, v, idx, gate_logit, n_sel, maskT, rows_ws, o, attn_lse, cs);
        return cuda_status(e);
    }
    return cuda_status(launch_fwd_simt(s, q, k, v, idx, gate_logit, n_sel, o, attn_lse, cs));
}

sas_status sas_gated_attn_bwd(const sas_desc* desc, const void* q, const void* k, const void* v, const void* o,
                              const void* dO, const float* attn_lse, const float* scores, const float* score_lse,
                              const int32_t* idx, const float* gate_logit, const int32_t* n_sel, void* dq,
                              void* dk, void* dv, float* dscores, void* ws, size_t ws_bytes_, void* stream) {
    Shape s;
    sas_status st = make_shape(desc, Kind::kTrain, &s);
    if (st != SAS_OK) return st;
    if (any_null(q, k, v, o, dO, attn_lse, scores, score_lse, idx, gate_logit, n_sel, dq, dk, dv, dscores))
        return SAS_ERR_INVALID_ARG;
    if (any_misaligned(q, k, v, o, dO, attn_lse, scores, score_lse, idx, gate_logit, n_sel, dq, dk, dv, dscores))
        return SAS_ERR_MISALIGNED;
    const TrainWs L = bwd_layout(s);
    if (ws == nullptr || ws_bytes_ < L.total) return SAS_ERR_WORKSPACE;
    if (!aligned16(ws)) return SAS_ERR_MISALIGNED;
    cudaStream_t cs = (cudaStream_t)stream;
    unsigned char* w = static_cast<unsigned char*>(ws);
    uint64_t* maskT = reinterpret_cast<uint64_t*>(w + L.maskT);
    float* Dd = reinterpret_cast<float*>(w + L.Dd);
    float* gsum = reinterpret_cast<float*>(w + L.gsum);
    float* dq_acc = s.dtype == SAS_DT_FP32 ? static_cast<float*>(dq) : reinterpret_cast<float*>(w + L.dq_acc);

    int* aborted = reinterpret_cast<int*>(w + L.flag);
    cudaError_t e = cudaMemsetAsync(aborted, 0, sizeof(int), cs);
    if (e == cudaSuccess) e = launch_sel_bitmap_T(s, idx, n_sel, maskT, cs);
    if (e == cudaSuccess) e = launch_bwd_rowdot(s, o, dO, Dd, dq_acc, cs);   // zeroes dq_acc too
    float* dk32 = nullptr;
    float* dv32 = nullptr;
    if (s.kvdiv > 1) {
        dk32 = reinterpret_cast<float*>(w + L.dkv32);
        dv32 = reinterpret_cast<float*>(w + L.dkv32 + align256(sizeof(float) * (size_t)s.B * s.Hkv * s.T * s.D));
    }
    if (e == cudaSuccess) {
        if (bwd_tc_supported(s))
            e = launch_bwd_tc(s, q, k, v, dO, attn_lse, Dd, idx, gate_logit, n_sel, maskT, w + L.stream, dq_acc, dk,
                              dv, dk32, dv32, gsum, aborted, cs);
        else
            e = launch_bwd_simt(s, q, k, v, dO, attn_lse, Dd, idx, gate_logit, n_sel, maskT, dq_acc, dk, dv, dk32,
                                dv32, gsum, cs);
    }
    if (e == cudaSuccess && s.kvdiv > 1) e = launch_reduce_dkv(s, dk32, dv32, dk, dv, cs);
    if (e == cudaSuccess && s.dtype != SAS_DT_FP32) e = launch_cast_dq(s, dq_acc, dq, aborted, cs);
    if (e == cudaSuccess) e = launch_dscore(s, scores, score_lse, idx, n_sel, gsum, dscores, aborted, cs);
    return cuda_status(e);
}

sas_status sas_sparse_decode(const sas_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                             int64_t cache_stride_tokens, const int32_t* idx, const float* gate_logit,
                             const int32_t* n_sel, void* o, void* ws, size_t ws_bytes_, void* stream) {
    Shape s;
    sas_status st = check_decode_args(desc, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o, &s);
    if (st != SAS_OK) return st;
    const size_t need = ws_bytes(SAS_OP_DECODE, s);
    if (ws == nullptr || ws_bytes_ < need) return SAS_ERR_WORKSPACE;
    if (!aligned16(ws)) return SAS_ERR_MISALIGNED;
    return cuda_status(launch_decode(s, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o,
                                     static_cast<float*>(ws), (cudaStream_t)stream));
}

sas_status sas_sparse_decode_paged(const sas_desc* desc, const void* q, const void* k_pages, const void* v_pages,
                                   int32_t num_pages, const int32_t* block_table, int32_t max_blocks,
                                   const int32_t* seq_lens, const int32_t* idx, const float* gate_logit,
                                   const int32_t* n_sel, void* o, void* ws, size_t ws_bytes_, void* stream) {
    Shape s;
    sas_status st = make_shape(desc, Kind::kDecode, &s);
    if (st != SAS_OK) return st;
    if (any_null(q, k_pages, v_pages, block_table, seq_lens, o)) return SAS_ERR_INVALID_ARG;
    if (idx != nullptr && any_null(gate_logit, n_sel)) return SAS_ERR_INVALID_ARG;
    if (num_pages < 1 || max_blocks < s.NB) return SAS_ERR_INVALID_ARG;
    if (!decode_paged_supported(s, num_pages)) return SAS_ERR_UNSUPPORTED;
    if (any_misaligned(q, k_pages, v_pages, block_table, seq_lens, o)) return SAS_ERR_MISALIGNED;
    if (idx != nullptr && any_misaligned(idx, gate_logit, n_sel)) return SAS_ERR_MISALIGNED;
    const size_t need = ws_bytes(SAS_OP_DECODE, s);
    if (ws == nullptr || ws_bytes_ < need) return SAS_ERR_WORKSPACE;
    if (!aligned16(ws)) return SAS_ERR_MISALIGNED;
    return cuda_status(launch_decode_paged(s, q, k_pages, v_pages, num_pages, block_table, max_blocks, seq_lens, idx,
                                           gate_logit, n_sel, o, static_cast<float*>(ws), (cudaStream_t)stream));
}

sas_status sas_block_scores_pooled(const sas_desc* desc, const void* q, const void* kbar,
                                   int64_t kbar_stride_blocks, float* scores, void* stream) {
    Shape s;
    sas_status st = make_shape(desc, Kind::kDecode, &s);
    if (st != SAS_OK) return st;
    if (any_null(q, kbar, scores)) return SAS_ERR_INVALID_ARG;
    if (kbar_stride_blocks < (int64_t)(s.q_offset / s.bs)) return SAS_ERR_INVALID_ARG;
    if (s.dtype != SAS_DT_BF16 || s.D != 128) return SAS_ERR_UNSUPPORTED;
    if (any_misaligned(q, kbar, scores)) return SAS_ERR_MISALIGNED;
    return cuda_status(launch_pooled_scores(s, q, kbar, kbar_stride_blocks, scores, (cudaStream_t)stream));
}

sas_status sas_sparse_decode_pooled(const sas_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                                    int64_t cache_stride_tokens, const void* kbar, int64_t kbar_stride_blocks,
                                    float* scores, int32_t* idx, float* gate_logit, float* score_lse,
                                    int32_t* n_sel, void* o, void* ws, size_t ws_bytes_, void* stream) {
    Shape s;
    sas_status st = check_decode_args(desc, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o, &s);
    if (st != SAS_OK) return st;
    if (any_null(kbar, scores, idx, score_lse)) return SAS_ERR_INVALID_ARG;
    if (kbar_stride_blocks < (int64_t)(s.q_offset / s.bs)) return SAS_ERR_INVALID_ARG;
    if (s.dtype != SAS_DT_BF16 || s.D != 128) return SAS_ERR_UNSUPPORTED;
    if (any_misaligned(kbar, scores, score_lse)) return SAS_ERR_MISALIGNED;
    const size_t need = ws_bytes(SAS_OP_DECODE, s);
    if (ws == nullptr || ws_bytes_ < need) return SAS_ERR_WORKSPACE;
    if (!aligned16(ws)) return SAS_ERR_MISALIGNED;
    cudaStream_t cs = (cudaStream_t)stream;
    cudaError_t e = launch_pooled_scores(s, q, kbar, kbar_stride_blocks, scores, cs);
    if (e == cudaSuccess) e = launch_block_topk(s, scores, nullptr, idx, gate_logit, score_lse, n_sel, cs);
    if (e == cudaSuccess)
        e = launch_decode(s, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o,
                          static_cast<float*>(ws), cs);
    return cuda_status(e);
}

// Diagnostics: kernels launched by this library since it was loaded (host
// count, incremented after each successful launch).
uint64_t sas_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

sas_status sas_kernel_timing(const char* names) {
    std::lock_guard<std::mutex> lk(g_tmu);
    if (names != nullptr) {
        for (const TimingRec& r : g_recs) {
            g_pool.push_back(r.a);
            g_pool.push_back(r.b);
        }
        g_recs.clear();
        g_timing_err = false;
        g_filter = std::strcmp(names, "*") == 0 ? std::string("*") : "," + std::string(names) + ",";
    }
    g_timing = names != nullptr;
    return SAS_OK;
}

sas_status sas_kernel_time(const char* kernel, double* total_ms, uint32_t* launches) {
    if (!kernel || !total_ms || !launches) return SAS_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_tmu);
    if (g_timing_err) return SAS_ERR_CUDA;
    double sum = 0.0;
    uint32_t n = 0;
    for (const TimingRec& r : g_recs) {
        if (std::strcmp(r.name, kernel) != 0) continue;
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            return SAS_ERR_CUDA;
        sum += ms;
        ++n;
    }
    *total_ms = sum;
    *launches = n;
    return SAS_OK;
}

// Diagnostics: number of bounded device-side waits that gave up since the
// library was loaded (0 in normal operation). Synchronises the device.
sas_status sas_device_timeouts(uint32_t* count) {
    if (!count) return SAS_ERR_INVALID_ARG;
    unsigned int c0 = 0, c2 = 0, c3 = 0;
    cudaError_t e = read_decode_timeouts(&c0);
    if (e == cudaSuccess) e = read_bwd_tc_timeouts(&c2);
    if (e == cudaSuccess) e = read_fwd_rows_timeouts(&c3);
    if (e != cudaSuccess) return SAS_ERR_CUDA;
    *count = c0 + c2 + c3;
    return SAS_OK;
}

sas_status sas_set_wait_limit(uint64_t ns) {
    const unsigned long long v = ns == 0 ? kDefaultWaitNs : (unsigned long long)ns;
    cudaError_t e = set_decode_wait_limit(v);
    if (e == cudaSuccess) e = set_bwd_tc_wait_limit(v);
    if (e == cudaSuccess) e = set_fwd_rows_wait_limit(v);
    return e == cudaSuccess ? SAS_OK : SAS_ERR_CUDA;
}

}  // extern "C"
