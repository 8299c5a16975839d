// kernels.h -- internal launchers of libsas (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sas.h"

struct CUtensorMap_st;   // cuda.h: CUtensorMap

namespace sas {

// Host-side count of kernels this library has launched (sas_kernel_launches).
void count_launches(unsigned n);

// While per-kernel timing is on (sas_kernel_timing), records a CUDA event on
// `st` at construction and another at destruction under `name`.
class KernelTimer {
public:
    KernelTimer(const char* name, cudaStream_t st);
    ~KernelTimer();
    KernelTimer(const KernelTimer&) = delete;
    KernelTimer& operator=(const KernelTimer&) = delete;

private:
    const char* name_;
    cudaStream_t st_;
    void* start_;
};

// Launch with programmatic stream serialization: the kernel may start while
// the kernel ahead of it in the stream is still running, and waits for it
// (pdl_wait) before it reads anything that earlier work writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Problem shape, validated and derived from sas_desc by the entry points.
struct Shape {
    // Hkv: selection groups per batch (KV heads, or query heads under
    // per-query-head selection), G: query heads per selection group (1 then);
    // Hkvp: KV heads of k/v/caches; kvdiv: selection groups per KV head.
    int B, T, q_offset, Hq, Hkv, G, D, bs, K;
    int Hkvp, kvdiv;
    int NB;        // ceil((q_offset + T) / bs): score columns per row
    int nT;        // T / bs (training only): query tiles per (b, kv head)
    float scale;   // softmax scale on q.k
    int dtype;     // sas_dtype
    int gate;      // sas_gate
    __host__ __device__ int64_t rows() const { return (int64_t)B * Hkv * T; }
    // (b, KV head) index of the K/V that selection group bg = b * Hkv + g reads
    __host__ __device__ int64_t kv_index(int64_t bg) const {
        return kvdiv == 1 ? bg : (bg / Hkv) * Hkvp + (bg % Hkv) / kvdiv;
    }
};

// K1: gate normaliser + hard top-K for every (b, kv head, t) row. `lens`
// (device, may be NULL): per-sequence cache lengths of decode rows (T = 1);
// row (b, g) then has floor((lens[b] - 1) / bs) candidates.
cudaError_t launch_block_topk(const Shape& s, const float* scores, const int32_t* lens, int32_t* idx,
                              float* gate_logit, float* score_lse, int32_t* n_sel, cudaStream_t st);
bool topk_row_supported(int64_t max_candidates);

// K1b: column-major selection bitmap maskT[b, g, j, tau] (bit r: query
// tau*bs + r kept block j). Requires training shapes (q_offset 0, T % bs 0).
cudaError_t launch_sel_bitmap_T(const Shape& s, const int32_t* idx, const int32_t* n_sel,
                                uint64_t* maskT, cudaStream_t st);

// Per-key-block token streams of the gathered-row kernels (stream.cu). For
// block (b, g, j): entries base[(b*Hkv+g)*NB+j] .. + count[...], each
// ent = {t, bits of the log-gate of j for t, slot of j in t's kept list, 0}
// and rv[e*rvs + h*vals + v] = row value v (v0, v1) of query head h of token t.
struct SelStream {
    int4* ent;
    float* rv;
    int* base;
    int* count;
    int* pre;       // [blocks, nT]: entries before query tile tau in block j's run (tau > j)
    int* counter;   // allocation counter, zeroed by launch_sel_stream
    int rvs;        // floats per entry in rv (G * vals rounded up to 4)
};
int sel_stream_rvs(const Shape& s, int vals);
int64_t sel_stream_capacity(const Shape& s);
size_t sel_stream_bytes(const Shape& s, int vals);
SelStream sel_stream_at(void* ws, const Shape& s, int vals);
cudaError_t launch_sel_stream(const Shape& s, const uint64_t* maskT, const int32_t* idx, const float* gl,
                              const int32_t* nsel, const float* v0, const float* v1, int vals, const SelStream& st,
                              cudaStream_t stream);

// Query-centric CUDA-core forward (fp32 and bf16).
cudaError_t launch_fwd_simt(const Shape& s, const void* q, const void* k, const void* v,
                            const int32_t* idx, const float* gate_logit, const int32_t* n_sel,
                            void* o, float* attn_lse, cudaStream_t st);
// The CUDA-core forward over the (b, kv head, t) rows list[0 .. *list_n)
// (device count); bf16, d 128, block 64.
cudaError_t launch_fwd_simt_rows(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                 const float* gl, const int32_t* nsel, const int32_t* list, const int32_t* list_n,
                                 void* o, float* lse, cudaStream_t st);

// 2D bf16 tensor map [rows x cols] with 64 x box_rows boxes, 128-byte swizzle.
bool encode_bf16_2d(::CUtensorMap_st* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// Tensor-core backward (tcgen05 + TMA + cp.async gathers): bf16, d = 128, block 64.
// ws (bwd_tc_ws_bytes) holds the per-block token streams it builds first.
bool bwd_tc_supported(const Shape& s);
size_t bwd_tc_ws_bytes(const Shape& s);
cudaError_t launch_bwd_tc(const Shape& s, const void* q, const void* k, const void* v, const void* dO,
                          const float* attn_lse, const float* Dd, const int32_t* idx, const float* gate_logit,
                          const int32_t* n_sel, const uint64_t* maskT, void* ws, float* dq_acc, void* dk, void* dv,
                          float* dk32, float* dv32, float* gsum, int* aborted, cudaStream_t st);

// Tensor-core forward over gathered rows (two passes + finalize): bf16, d = 128, block 64.
bool fwd_rows_supported(const Shape& s);
size_t fwd_rows_ws_bytes(const Shape& s);
cudaError_t launch_fwd_rows(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                            const float* gate_logit, const int32_t* n_sel, const uint64_t* maskT, void* ws, void* o,
                            float* attn_lse, cudaStream_t st);

// Backward pieces.
// D = rowsum(o * dO) per query-head row; also zeroes the fp32 dq accumulator [rows, d].
cudaError_t launch_bwd_rowdot(const Shape& s, const void* o, const void* dO, float* Dd, float* dq_acc,
                              cudaStream_t st);
cudaError_t launch_bwd_simt(const Shape& s, const void* q, const void* k, const void* v, const void* dO,
                            const float* attn_lse, const float* Dd, const int32_t* idx,
                            const float* gate_logit, const int32_t* n_sel, const uint64_t* maskT,
                            float* dq_acc, void* dk, void* dv, float* dk32, float* dv32, float* gsum,
                            cudaStream_t st);
// Per-query-head selection (s.kvdiv > 1): the backward kernels write fp32 dK, dV
// per selection group into dk32/dv32 [B * Hkv, T, d] (NULL otherwise); this
// sums the kvdiv groups of each KV head into dk, dv [B, Hkvp, T, d] (s.dtype).
cudaError_t launch_reduce_dkv(const Shape& s, const float* dk32, const float* dv32, void* dk, void* dv,
                              cudaStream_t st);
// fp32 dq accumulator -> bf16 dq (bf16 shapes only; fp32 accumulates in place).
// `aborted` (device flag, may be NULL): when set, dq is written as NaN.
cudaError_t launch_cast_dq(const Shape& s, const float* dq_acc, void* dq, const int* aborted, cudaStream_t st);
// Score gradient; `aborted` (device flag, may be NULL): when set, every row is NaN.
cudaError_t launch_dscore(const Shape& s, const float* scores, const float* score_lse,
                          const int32_t* idx, const int32_t* n_sel, const float* gsum, float* dscores,
                          const int* aborted, cudaStream_t st);

// Pooled-key block scores of decode rows (bf16, d 128): scores[b, g, 0, j] =
// mean_G(q) . kbar[b, g, j] for j < C, 0 for C <= j < NB; kbar [B, Hkv,
// kstride, d].
cudaError_t launch_pooled_scores(const Shape& s, const void* q, const void* kbar, int64_t kstride, float* scores,
                                 cudaStream_t st);

// Decode argument checks shared by the decode entry points (sas_api.cu).
sas_status check_decode_args(const sas_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                             int64_t cache_stride_tokens, const int32_t* idx, const float* gate_logit,
                             const int32_t* n_sel, const void* o, Shape* s);

// Decode.
struct DecodePlan {
    int bpc;      // blocks per CTA
    int splits;   // CTAs per (b, kv head)
};
DecodePlan decode_plan(const Shape& s, bool dense);
size_t decode_ws_bytes(const Shape& s);
cudaError_t launch_decode(const Shape& s, const void* q, const void* kc, const void* vc, int64_t stride,
                          const int32_t* idx, const float* gate_logit, const int32_t* n_sel, void* o,
                          float* part, cudaStream_t st);
// Paged cache (bf16, d 128, block 64): pools [num_pages, Hkv, 64, d], block j
// of sequence b in page table[b * max_blocks + j], cache length lens[b].
bool decode_paged_supported(const Shape& s, int64_t num_pages);
cudaError_t launch_decode_paged(const Shape& s, const void* q, const void* kp, const void* vp, int num_pages,
                                const int32_t* table, int max_blocks, const int32_t* lens, const int32_t* idx,
                                const float* gate_logit, const int32_t* n_sel, void* o, float* part,
                                cudaStream_t st);

}  // namespace sas
