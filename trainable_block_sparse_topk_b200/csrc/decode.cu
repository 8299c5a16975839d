// decode.cu -- budgeted sparse decode (and dense decode) over a KV cache.
//
// One new token per (batch, query head) at position N - 1 attends the K kept
// historical blocks of its KV group plus the causal current block
// (SAS study note 3-7 inference path, steps 2-4). With no selection it attends
// every token [0, N) with no gate: the dense comparison of study note 5-6.
//
// bf16, d 128, block 64 (the tensor-core path, decode_flat_kernel): persistent
// CTAs, one per SM, share out every (b, kv head)'s block list evenly, stream
// the blocks by TMA and merge the per-CTA partials in the last CTA to finish
// each group -- one launch per call. Other shapes and fp32 (CUDA cores,
// decode_partial_kernel): the block list of each (b, kv head) is cut into
// `splits` chunks of `bpc` blocks; one CTA per chunk streams its blocks
// through two shared memory stages, one bulk async copy per tensor and block
// (K and V rows of a block are contiguous in the cache), writes an
// unnormalised partial (m, l, o) for the G heads, and a second kernel merges
// the partials by log-sum-exp.
#include <algorithm>
#include <mutex>

#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sas {

namespace {

constexpr int kDecThreads = 256;

// Flat item split of the tensor-core decode: nblk items per (b, kv head)
// group, W items in all, ncta CTAs, each owning per or per + 1 of them.
struct FlatPlan {
    int64_t W;
    int nblk;
    int ncta;
    int64_t per, rem;
};

struct DecArgs {
    Shape sh;
    const void* q;
    const void* kc;
    const void* vc;
    int64_t stride;      // cache tokens per (b, kv head)
    const int32_t* idx;  // nullptr: dense
    const float* gl;
    const int32_t* nsel;
    float* part;         // [B*Hkv][splits][G][D + 2]: o (unnormalised), m (log2 units), l
    void* o;             // [B, Hq, D] output
    int bpc;
    int splits;
    FlatPlan fp;         // tensor-core path: item split
    int* fin;            // tensor-core path: [B*Hkv] records written per group, zeroed per call
    int cs;              // tensor-core path: 0 = flat item split; >= 1: a cluster of cs CTAs per group
    // paged cache (tensor-core path): block j of sequence b is page
    // table[b * max_blocks + j] of the pools kc/vc [num_pages, Hkv, BS, D];
    // NULL table: the contiguous cache [B, Hkv, stride, D]
    const int32_t* table;
    int max_blocks;
    int num_pages;
    const int32_t* lens; // [B] cache length of each sequence (new token included); NULL: q_offset + 1
};

template <typename T, int D, int BS>
constexpr size_t dec_stage_bytes() { return (size_t)2 * BS * D * sizeof(T); }

// Region 0 holds the two stages while streaming and the cross-key-group
// reduction buffer [NKG][GMAX][D] afterwards.
template <typename T, int D, int GMAX, int BS>
constexpr size_t dec_region0_bytes() {
    constexpr size_t stages = 2 * dec_stage_bytes<T, D, BS>();
    constexpr size_t red = (size_t)(kDecThreads / (D * (int)sizeof(T) / 16)) * GMAX * D * sizeof(float);
    return stages > red ? stages : red;
}

template <typename T, int D, int GMAX, int BS>
constexpr size_t dec_smem_bytes() {
    // region 0; q [GMAX][D]; p [BS][GMAX]; m,l,corr [GMAX]; 2 mbarriers; flag.
    return dec_region0_bytes<T, D, GMAX, BS>() + sizeof(float) * (GMAX * D + BS * GMAX + 3 * GMAX + 1) + 2 * 8 +
           16;
}

template <typename T, int D, int GMAX, int BS>
__global__ void __launch_bounds__(kDecThreads)
decode_partial_kernel(DecArgs a) {
    constexpr int VE = vec16<T>();             // elements per 16-byte chunk
    constexpr int CPR = D * (int)sizeof(T) / 16;  // chunks per row
    constexpr int NKG = kDecThreads / CPR;     // key groups in the PV phase
    constexpr int CPT = CPR / 8;               // chunks per thread in the score phase
    constexpr size_t STAGE = dec_stage_bytes<T, D, BS>();
    constexpr size_t HALF = STAGE / 2;
    static_assert(CPR % 8 == 0 && kDecThreads % CPR == 0, "layout");

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* stage_base = smem;
    constexpr size_t R0 = dec_region0_bytes<T, D, GMAX, BS>();
    float* qs = reinterpret_cast<float*>(smem + R0);          // [GMAX][D], pre-scaled to log2 units
    float* ps = qs + GMAX * D;                                 // [BS][GMAX]
    float* st_m = ps + BS * GMAX;
    float* st_l = st_m + GMAX;
    float* st_c = st_l + GMAX;
    uint64_t* bars = reinterpret_cast<uint64_t*>(st_c + GMAX + (GMAX & 1));
    int* flag = reinterpret_cast<int*>(bars + 2);

    const Shape& sh = a.sh;
    const int G = sh.G;
    const int tid = threadIdx.x;
    const int split = blockIdx.x % a.splits;
    const int64_t bg = blockIdx.x / a.splits;
    const int b = (int)(bg / sh.Hkv), g = (int)(bg % sh.Hkv);
    const int64_t N = (int64_t)sh.q_offset + 1;
    const int C = (int)(sh.q_offset / BS);
    const bool dense = a.idx == nullptr;
    // a kept count outside [0, min(K, C)] would read past the row: clamp it
    const int n = dense ? C : min(max(a.nsel[bg], 0), min(sh.K, C));
    const int nblk = n + 1;
    const int p0 = split * a.bpc;
    const int p1 = min(p0 + a.bpc, nblk);
    const int cnt = max(p1 - p0, 0);

    const T* kc = static_cast<const T*>(a.kc) + sh.kv_index(bg) * a.stride * D;
    const T* vc = static_cast<const T*>(a.vc) + sh.kv_index(bg) * a.stride * D;

    // An index outside [0, C) is not a valid selection: such a block is
    // skipped (no copy, no keys) rather than read out of bounds.
    auto block_of = [&](int pos) -> int {
        if (dense) return pos;
        if (pos >= n) return C;
        const int j = a.idx[bg * sh.K + pos];
        return ((unsigned)j < (unsigned)C) ? j : -1;
    };
    auto ntok_of = [&](int j) -> int { return j < 0 ? 0 : (j == C ? (int)(N - (int64_t)C * BS) : BS); };
    auto issue = [&](int i) {  // thread 0 only: block p0 + i into stage i & 1
        const int j = block_of(p0 + i);
        const uint32_t bytes = (uint32_t)ntok_of(j) * D * (uint32_t)sizeof(T);
        unsigned char* dst = stage_base + (size_t)(i & 1) * STAGE;
        mbar_arrive_expect_tx(&bars[i & 1], 2 * bytes);
        if (bytes > 0) {
            bulk_g2s(dst, kc + (int64_t)j * BS * D, bytes, &bars[i & 1]);
            bulk_g2s(dst + HALF, vc + (int64_t)j * BS * D, bytes, &bars[i & 1]);
        }
    };

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < cnt && i < 2; ++i) issue(i);
    }
    const float qscale = sh.scale * kLog2e;
    const T* qg = static_cast<const T*>(a.q) + ((int64_t)b * sh.Hq + (int64_t)g * G) * D;
    for (int e = tid; e < GMAX * D; e += kDecThreads) qs[e] = e < G * D ? Elem<T>::to_f(qg[e]) * qscale : 0.f;
    if (tid < GMAX) { st_m[tid] = -INFINITY; st_l[tid] = 0.f; st_c[tid] = 1.f; }

    // PV-phase ownership: chunk c (VE dims) of keys kg, kg + NKG, ...
    const int pc = tid % CPR, kg = tid / CPR;
    float acc[GMAX][VE];
#pragma unroll
    for (int h = 0; h < GMAX; ++h)
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[h][e] = 0.f;
    // score-phase ownership: key sk = tid / 8 (+32 per round), chunks c8 + 8i
    const int c8 = tid & 7;

    int failed = -1;
    for (int i = 0; i < cnt; ++i) {
        const int j = block_of(p0 + i);
        const int ntok = ntok_of(j);
        const float lg = (!dense && p0 + i < n) ? a.gl[bg * sh.K + p0 + i] * kLog2e : 0.f;
        if (tid == 0) flag[0] = mbar_wait_bounded(&bars[i & 1], (uint32_t)((i >> 1) & 1)) ? 1 : 0;
        __syncthreads();
        if (!flag[0]) { failed = i; break; }
        const T* Ks = reinterpret_cast<const T*>(stage_base + (size_t)(i & 1) * STAGE);
        const T* Vs = reinterpret_cast<const T*>(stage_base + (size_t)(i & 1) * STAGE + HALF);

        // ---- scores: 8 threads per key, reduced by shuffles ----
#pragma unroll
        for (int r = 0; r < BS / 32; ++r) {
            const int sk = (tid >> 3) + 32 * r;
            float s[GMAX];
#pragma unroll
            for (int h = 0; h < GMAX; ++h) s[h] = 0.f;
            if (sk < ntok) {
#pragma unroll
                for (int ci = 0; ci < CPT; ++ci) {
                    const int c = c8 + 8 * ci;
                    float kv[VE];
                    load_vec<T, VE>(Ks + sk * D + c * VE, kv);
#pragma unroll
                    for (int h = 0; h < GMAX; ++h) {
                        if (h < G) {
#pragma unroll
                            for (int e = 0; e < VE; ++e) s[h] = fmaf(qs[h * D + c * VE + e], kv[e], s[h]);
                        }
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                s[h] += __shfl_xor_sync(0xffffffffu, s[h], 1);
                s[h] += __shfl_xor_sync(0xffffffffu, s[h], 2);
                s[h] += __shfl_xor_sync(0xffffffffu, s[h], 4);
            }
            if (c8 == 0 && sk < BS) {
#pragma unroll
                for (int h = 0; h < GMAX; ++h) ps[sk * GMAX + h] = sk < ntok ? s[h] + lg : -INFINITY;
            }
        }
        __syncthreads();

        // ---- online softmax: warp h owns head h ----
        {
            const int w = tid >> 5, lane = tid & 31;
            if (w < G) {
                float x[BS / 32];
                float mx = -INFINITY;
#pragma unroll
                for (int r = 0; r < BS / 32; ++r) { x[r] = ps[(lane + 32 * r) * GMAX + w]; mx = fmaxf(mx, x[r]); }
                mx = warp_max(mx);
                const float mo = st_m[w];
                const float mn = fmaxf(mo, mx);
                float sum = 0.f;
#pragma unroll
                for (int r = 0; r < BS / 32; ++r) {
                    const float pv = mn == -INFINITY ? 0.f : exp2f(x[r] - mn);
                    ps[(lane + 32 * r) * GMAX + w] = pv;
                    sum += pv;
                }
                sum = warp_sum(sum);
                if (lane == 0) {
                    const float corr = mo == -INFINITY ? 0.f : exp2f(mo - mn);
                    st_c[w] = corr;
                    st_l[w] = st_l[w] * corr + sum;
                    st_m[w] = mn;
                }
            }
        }
        __syncthreads();

        // ---- o = o * corr + P V ----
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            const float c = st_c[h];
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[h][e] *= c;
        }
        for (int key = kg; key < ntok; key += NKG) {
            float vv[VE];
            load_vec<T, VE>(Vs + key * D + pc * VE, vv);
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                const float pk = ps[key * GMAX + h];
#pragma unroll
                for (int e = 0; e < VE; ++e) acc[h][e] = fmaf(pk, vv[e], acc[h][e]);
            }
        }
        __syncthreads();   // every thread is done with this stage and with ps
        if (tid == 0 && i + 2 < cnt) issue(i + 2);
    }

    if (failed >= 0) {
        // A copy never completed: wait (bounded) for the copies still in
        // flight into this CTA's shared memory, then leave NaN partials so the
        // result is visibly invalid.
        if (tid == 0) {
            for (int i = failed; i < cnt && i < failed + 2; ++i)
                mbar_wait_bounded(&bars[i & 1], (uint32_t)((i >> 1) & 1));
        }
        __syncthreads();
        float* rec = a.part + (bg * a.splits + split) * (int64_t)G * (D + 2);
        for (int e = tid; e < G * (D + 2); e += kDecThreads) rec[e] = __int_as_float(0x7fc00000);
        return;
    }

    // ---- reduce acc over the NKG key groups (reusing the stage buffers) ----
    float* red = reinterpret_cast<float*>(stage_base);   // [NKG][GMAX][D], fits region 0
#pragma unroll
    for (int h = 0; h < GMAX; ++h)
#pragma unroll
        for (int e = 0; e < VE; ++e) red[((size_t)kg * GMAX + h) * D + pc * VE + e] = acc[h][e];
    __syncthreads();
    float* rec = a.part + (bg * a.splits + split) * (int64_t)G * (D + 2);
    for (int e = tid; e < G * D; e += kDecThreads) {
        const int h = e / D, d = e % D;
        float s = 0.f;
#pragma unroll 4
        for (int x = 0; x < NKG; ++x) s += red[((size_t)x * GMAX + h) * D + d];
        rec[h * (D + 2) + d] = s;
    }
    if (tid < G) {
        rec[tid * (D + 2) + D] = st_m[tid];
        rec[tid * (D + 2) + D + 1] = st_l[tid];
    }
}

// ---------------------------------------------------------------------------
// Tensor-core decode (bf16, d = 128, block 64, G <= 8): persistent CTAs over a
// flat list of work items.
//
// Item i is position p = i % nblk of group bg = i / nblk, the (b, kv head)
// block lists laid end to end. Sparse: p < n is the p-th kept block, the last
// position (nblk - 1 = min(K, C)) is the causal current block, and positions
// in between (a row that kept fewer than min(K, C) blocks) are empty. Dense:
// p is the block index itself, the last one being the current block.
// CTA c takes the contiguous items [start(c), start(c + 1)), an even share of
// all of them, so a group's list may be cut between neighbouring CTAs and a
// CTA may finish one group and start the next. For every group it touches, a
// CTA writes one unnormalised partial (m, l, O of the G heads) as record
// c + bg (unique: the groups of CTA c + 1 start where those of CTA c end).
// The CTA that completes a group last (an atomic ticket per group) merges the
// group's records by log-sum-exp and writes o: one launch per call.
//
// Roles (224 threads): warp 0 resolves the items' block indices, log-gates
// and cache rows 32 at a time and moves each block's K and V rows into a
// kFlatStages ring by TMA (two 64-column boxes per tensor, 128-byte swizzle, no
// multicast); warps 1-6 form three pairs, each pair taking every third item
// and owning two stages, each warp of a pair taking 32 of the block's 64 keys
// (an mma.sync chain has little parallelism of its own, so six half-blocks are
// computed at once) and running them on mma.sync m16n8k16:
//   S^T = K q^T   (M = 16 keys, N = 8 heads, K = 16 dims; 2 x 8 MMAs per warp)
//   online softmax per head in log2 units (scale applied in fp32 after the MMA)
//   O^T += V^T P^T (M = 16 dims, N = 8 heads, K = 16 keys; 8 x 2 MMAs per warp)
// K rows come through ldmatrix, V rows through ldmatrix.trans, and the P tile
// (keys x heads, accumulator layout) becomes the B operand by movmatrix.trans.
// Rows of the current block at or after the new token may hold anything in the
// cache: their scores are replaced by -inf and their V rows zeroed in shared
// memory before the product. At the end of each group the consumers merge
// their (m, l, O) through shared memory.
constexpr int kFlatStages = 6;
constexpr int kCons = 3;                 // consumer pairs: item i goes to pair i mod kCons
constexpr int kConsWarps = 2 * kCons;    // each pair splits a block's 64 keys, 32 per warp
constexpr int kFlatThreads = 32 * (1 + kConsWarps);
// Stage s always holds items of pair s mod kCons, so each stage's barrier
// phases are waited on by the same two warps, each in order (a warp of another
// pair could poll a phase ahead of the current one and see an older phase of
// the same parity).
static_assert(kFlatStages % kCons == 0, "every stage must belong to one consumer pair");
constexpr uint32_t kItemBytes = 32768;   // K box 0 | K box 1 | V box 0 | V box 1, 8 KiB each
constexpr int kMaxDecodeCtas = 160;     // grid bound (one CTA per SM)
constexpr int kRecF = 132;              // floats per head in a record: O[128], m, l, 2 pad (16-byte rows)
constexpr int kMaxRecs = 64;            // records of one group (CTAs sharing it), bounded by the plan
// One consumer's state in shared memory: m[8], l[8], then O[8 heads][kXchRow]
// (128 dims + 4 pad: the publishing lanes (8 dims x 4 head pairs) hit 32
// distinct banks, and a warp reading one head's row takes whole 16-byte runs).
constexpr int kXchRow = 132;
constexpr int kXchF = 16 + 8 * kXchRow;
constexpr int kMaxCluster = 8;          // portable cluster size
constexpr unsigned long long kRecvFloorNs = 10000000ull;   // shortest wait of a cluster leader for the partials

// Item split: CTA c owns [flat_start(c), flat_start(c + 1)).
__host__ __device__ __forceinline__ int64_t flat_start(const FlatPlan& f, int64_t c) {
    return c * f.per + (c < f.rem ? c : f.rem);
}
// The CTA that owns item i.
__host__ __device__ __forceinline__ int64_t flat_owner(const FlatPlan& f, int64_t i) {
    const int64_t big = f.rem * (f.per + 1);
    return i < big ? i / (f.per + 1) : f.rem + (i - big) / f.per;
}

struct FlatSmem {
    static constexpr uint32_t kBar = kFlatStages * kItemBytes;        // full[S], empty[S]
    static constexpr uint32_t kMisc = kBar + 16 * kFlatStages;        // i32 abort flag; mbarrier rcv at + 8
    static constexpr uint32_t kBlk = kMisc + 16;                      // i32 [S]: keys of the stage's item (0: none)
    static constexpr uint32_t kLg = kBlk + 4 * kFlatStages;           // f32 [S]: its log-gate (log2 units)
    static constexpr uint32_t kXch = (kLg + 4 * kFlatStages + 15) & ~15u;   // per consumer: m[8], l[8], O[8][kXchRow]
    static constexpr uint32_t kLast = kXch + 4 * kConsWarps * kXchF;  // i32: this CTA merges the group
    // flat split: f32 m, l, weight [kMaxRecs][8] each (the last CTA's merge);
    // cluster: this CTA's partial, G rows of kRecF floats (O, m, l) read by the leader
    static constexpr uint32_t kMerge = kLast + 16;
    static constexpr uint32_t kTotal = kMerge + 3 * 4 * kMaxRecs * 8;
};
static_assert(3 * kMaxRecs * 8 >= 8 * kRecF, "the cluster partial fits the merge area");
static_assert(FlatSmem::kTotal + 1024 <= 232448, "shared memory of one CTA");

__device__ __forceinline__ uint32_t sw_addr(uint32_t box, int row, int chunk) {
    return box + (uint32_t)row * 128u + (uint32_t)((chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The address of this CTA's shared-memory location `a` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
// Asynchronous 16-byte store into another CTA's shared memory that counts its
// bytes on that CTA's mbarrier (both addresses in the cluster window).
__device__ __forceinline__ void st_async_f32x4(uint32_t a, float4 v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
                 ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar) : "memory");
}
// Bounded wait, with cluster-scope acquire, for the partials that the other
// CTAs of the cluster store into this CTA's shared memory.
__device__ __forceinline__ bool rcv_wait(uint64_t* bar, unsigned long long lim) {
    const uint64_t t0 = global_ns();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n"
            " selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done) : "r"(smem_u32(bar)) : "memory");
        if (done) return true;
        if (global_ns() - t0 > lim) return false;
    }
}

// kClu = false: flat item split over persistent CTAs, records merged by the
// last CTA of each group. kClu = true: a cluster of a.cs CTAs per group, each
// taking an even share of the group's items; the cluster's leader (rank 0)
// reads the other CTAs' partials from their shared memory and writes o.
template <bool kClu>
__global__ void __launch_bounds__(kFlatThreads, 1)
decode_flat_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ DecArgs a) {
    constexpr int D = 128, BS = 64;
    using L = FlatSmem;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* empty = full + kFlatStages;
    volatile int* abort = reinterpret_cast<volatile int*>(sm + L::kMisc);
    int* s_ntok = reinterpret_cast<int*>(sm + L::kBlk);
    float* s_lg = reinterpret_cast<float*>(sm + L::kLg);
    float* xch = reinterpret_cast<float*>(sm + L::kXch);
    volatile int* s_last = reinterpret_cast<volatile int*>(sm + L::kLast);
    float* s_mg = reinterpret_cast<float*>(sm + L::kMerge);
    float* s_lg2 = s_mg + kMaxRecs * 8;
    float* s_wg = s_lg2 + kMaxRecs * 8;

    const Shape& sh = a.sh;
    const FlatPlan& fp = a.fp;
    const int G = sh.G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t cta = blockIdx.x;
    const int nblk = fp.nblk;
    int64_t i0, i1;
    uint32_t rank = 0;
    if constexpr (kClu) {
        // grid = groups x cs, cluster dims (cs, 1, 1). The leader (rank 0) takes
        // the first n0 items of group bg (n0 = nblk / 2 for cs = 2, at most
        // kCons for larger clusters, all of them for cs = 1); ranks 1 .. cs - 1
        // share the rest evenly.
        rank = cluster_rank();
        const int cs = a.cs;
        const int64_t bg = cta / cs;
        const int n0 = cs == 1 ? nblk : cs == 2 ? nblk / 2 : min(kCons, nblk / cs);
        if (rank == 0) {
            i0 = bg * nblk;
            i1 = i0 + n0;
        } else {
            const int rest = nblk - n0, per = rest / (cs - 1), rem = rest % (cs - 1), r = (int)rank - 1;
            i0 = bg * nblk + n0 + (int64_t)r * per + min(r, rem);
            i1 = i0 + per + (r < rem ? 1 : 0);
        }
    } else {
        i0 = flat_start(fp, cta);
        i1 = flat_start(fp, cta + 1);
    }
    const int nitems = (int)(i1 - i0);
    const int64_t N = (int64_t)sh.q_offset + 1;       // the longest cache length
    const bool dense = a.idx == nullptr;

    uint64_t* rcv = reinterpret_cast<uint64_t*>(sm + L::kMisc + 8);
    const bool clu = kClu && a.cs > 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kFlatStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 2);   // both warps of the owning pair
        }
        mbar_init(rcv, 1);
        // the leader expects G rows of kRecF floats from each other CTA
        if (clu && rank == 0) mbar_arrive_expect_tx(rcv, (uint32_t)((a.cs - 1) * G * kRecF * 4));
        *abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // Every CTA's barriers are initialised before any CTA of the cluster
    // stores into the leader (the senders wait on this arrival before storing).
    if (clu) cluster_arrive_relaxed();
    // Stage ring: a cluster leader with cs >= 4 takes at most kCons items and
    // uses stages 0 .. kCons - 1 only; the rest receives the other partials.
    const int nst = (clu && a.cs >= 4 && rank == 0) ? kCons : kFlatStages;
    // Launched right behind the top-K, this CTA may already be running:
    // everything below reads what earlier kernels wrote.
    pdl_wait();

    if (warp == 0) {
        // ---- producer ----
        if (lane == 0) {
            tc::prefetch_tmap(&tm_k);
            tc::prefetch_tmap(&tm_v);
        }
        int issued = 0;
        bool stop = false;
        for (int base = 0; base < nitems && !stop; base += 32) {
            // lane l resolves item base + l: its block (-1: empty) and log-gate
            // lane l resolves item base + l: its keys (0: nothing to load), its
            // log-gate and the first cache row of its block
            int ntl = 0, rowl = 0;
            float lgl = 0.f;
            if (base + lane < nitems) {
                const int64_t i = i0 + base + lane;
                const int64_t bg = i / nblk;
                const int p = (int)(i - bg * nblk);
                const int b = (int)(bg / sh.Hkv), g = (int)(bg - (int64_t)b * sh.Hkv);
                const int64_t Nb = a.lens == nullptr ? N : min(max((int64_t)a.lens[b], (int64_t)1), N);
                const int Cb = (int)((Nb - 1) / BS);   // this sequence's current block
                int j = -1;
                // the kept index, its log-gate and the kept count are loaded together
                // (p < nblk - 1 <= K keeps the first two inside the row)
                int jj = -1, ns = 0;
                float gv = 0.f;
                if (!dense && p < nblk - 1) {
                    jj = a.idx[bg * sh.K + p];
                    gv = a.gl[bg * sh.K + p];
                    ns = a.nsel[bg];
                }
                if (dense) {
                    j = p <= Cb ? p : -1;
                } else if (p == nblk - 1) {
                    j = Cb;
                } else if (p < min(max(ns, 0), min(sh.K, Cb)) && (unsigned)jj < (unsigned)Cb) {
                    // a count outside [0, min(K, C)] is clamped; an index outside [0, C) skipped
                    j = jj;
                    lgl = gv * kLog2e;
                }
                if (j >= 0) {
                    if (a.table == nullptr) {
                        ntl = j == Cb ? (int)(Nb - (int64_t)Cb * BS) : BS;
                        rowl = (int)(sh.kv_index(bg) * a.stride + (int64_t)j * BS);
                    } else {
                        const int page = a.table[(int64_t)b * a.max_blocks + j];
                        if ((unsigned)page < (unsigned)a.num_pages) {   // an invalid page is skipped
                            ntl = j == Cb ? (int)(Nb - (int64_t)Cb * BS) : BS;
                            rowl = (page * sh.Hkvp + g / sh.kvdiv) * BS;
                        }
                    }
                }
            }
            const int cnt = min(32, nitems - base);
            for (int k = 0; k < cnt; ++k) {
                const int li = base + k;
                const int nt = __shfl_sync(0xffffffffu, ntl, k);
                const int row = __shfl_sync(0xffffffffu, rowl, k);
                const float lg = __shfl_sync(0xffffffffu, lgl, k);
                int fail = 0;
                if (lane == 0) {
                    const int s = li % nst;
                    if (li >= nst && !tc::wait_bar(&empty[s], (uint32_t)(((li / nst) - 1) & 1), abort)) {
                        fail = 1;
                    } else {
                        s_ntok[s] = nt;
                        s_lg[s] = lg;
                        if (nt == 0) {
                            tc::mbar_arrive(&full[s]);
                        } else {
                            mbar_arrive_expect_tx(&full[s], kItemBytes);
                            unsigned char* st = sm + s * kItemBytes;
                            tc::tma_load_2d(st, &tm_k, 0, row, &full[s]);
                            tc::tma_load_2d(st + 8192, &tm_k, 64, row, &full[s]);
                            tc::tma_load_2d(st + 16384, &tm_v, 0, row, &full[s]);
                            tc::tma_load_2d(st + 24576, &tm_v, 64, row, &full[s]);
                        }
                        ++issued;
                    }
                }
                if (__shfl_sync(0xffffffffu, fail, 0)) { stop = true; break; }
            }
        }
        if (lane == 0 && stop) {
            // let the copies already started land before the CTA exits
            for (int li = max(0, issued - nst); li < issued; ++li)
                tc::drain_wait(&full[li % nst], (uint32_t)((li / nst) & 1));
        }
        return;
    }

    // ---- consumers: warps 1 + 2c and 2 + 2c (pair c) take the CTA-local items
    // c, c + kCons, ...; the first warp of a pair takes keys 0-31 of each
    // block, the second keys 32-63, each with its own online-softmax state ----
    const int cw = warp - 1;
    const int pair = cw >> 1, hf = cw & 1;
    const int gq = lane >> 2, tq = lane & 3;
    const float qk = sh.scale * kLog2e;
    const uint32_t sbase = smem_u32(sm);
    bool ok = true;
    for (int64_t seg = i0; seg < i1;) {
        const int64_t bg = seg / nblk;
        const int64_t seg_end = min(i1, (bg + 1) * nblk);
        const int b = (int)(bg / sh.Hkv), g = (int)(bg % sh.Hkv);
        // q^T as the B operand: b0 = q[head gq][16 ks + 2 tq, +1], b1 = the same + 8
        uint32_t qb[8][2];
        {
            const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) + ((int64_t)b * sh.Hq + (int64_t)g * G) * D;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                if (gq < G) {
                    qb[ks][0] = *reinterpret_cast<const uint32_t*>(qg + gq * D + 16 * ks + 2 * tq);
                    qb[ks][1] = *reinterpret_cast<const uint32_t*>(qg + gq * D + 16 * ks + 2 * tq + 8);
                } else {
                    qb[ks][0] = qb[ks][1] = 0u;
                }
            }
        }
        float o[8][4];          // O^T: m-tile of 16 dims, (dim gq | gq+8) x (heads 2tq, 2tq+1)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;
        float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};   // heads 2tq, 2tq+1

        for (int64_t i = seg + (pair - (int)((seg - i0) % kCons) + kCons) % kCons; i < seg_end; i += kCons) {
            const int li = (int)(i - i0);
            const int s = li % nst;
            if (ok && !tc::warp_wait_bar(&full[s], (uint32_t)((li / nst) & 1), abort)) ok = false;
            const int ntok = ok ? s_ntok[s] : 0;
            if (ntok > 0) {
                const uint32_t kb0 = sbase + s * kItemBytes, kb1 = kb0 + 8192, vb0 = kb0 + 16384, vb1 = kb0 + 24576;
                if (ntok < 32 * hf + 32) {   // the current block: clear this half's V rows >= ntok (128 bytes per row and box)
                    unsigned char* v0p = sm + s * kItemBytes + 16384;
                    for (int e = max(ntok, 32 * hf) * 8 + lane; e < (32 * hf + 32) * 8; e += 32) {
                        reinterpret_cast<uint4*>(v0p)[e] = make_uint4(0, 0, 0, 0);
                        reinterpret_cast<uint4*>(v0p + 8192)[e] = make_uint4(0, 0, 0, 0);
                    }
                    __syncwarp();
                }
                const float lg = s_lg[s];
                // ---- S^T = K q^T over this warp's 32 keys (m-tiles 2 hf, 2 hf + 1) ----
                float sc[2][4];
#pragma unroll
                for (int m2 = 0; m2 < 2; ++m2) {
                    const int mt = 2 * hf + m2;
#pragma unroll
                    for (int e = 0; e < 4; ++e) sc[m2][e] = 0.f;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        // matrices: (keys +0..7, dims +0..7), (keys +8..15, dims +0..7), (keys +0..7, dims +8..15), (keys +8.., dims +8..)
                        const int key = 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
                        const int chunk = 2 * ks + (lane >> 4);
                        const uint32_t addr = sw_addr(chunk < 8 ? kb0 : kb1, key, chunk & 7);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(addr, a0, a1, a2, a3);
                        mma_bf16(sc[m2], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                    }
                }
                // ---- online softmax (heads 2tq, 2tq+1; keys 16 mt + gq (+8)) ----
                float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int m2 = 0; m2 < 2; ++m2)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = 16 * (2 * hf + m2) + gq + (e >> 1) * 8;
                        const float v = key < ntok ? fmaf(sc[m2][e], qk, lg) : -INFINITY;
                        sc[m2][e] = v;
                        mx[e & 1] = fmaxf(mx[e & 1], v);
                    }
                float corr[2], psum[2] = {0.f, 0.f};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 4));
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 8));
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
                    const float mn = fmaxf(mrun[h], mx[h]);
                    corr[h] = mrun[h] == -INFINITY ? 0.f : exp2f(mrun[h] - mn);
                    mrun[h] = mn;
                }
                uint32_t pb[2][2];   // P^T as B operand per k-step (16 keys)
#pragma unroll
                for (int m2 = 0; m2 < 2; ++m2) {
                    float p[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float m = mrun[e & 1];
                        p[e] = m == -INFINITY ? 0.f : exp2f(sc[m2][e] - m);
                        psum[e & 1] += p[e];
                    }
                    pb[m2][0] = movm_t(pack_bf16(p[0], p[1]));   // keys 16 mt + 0..7
                    pb[m2][1] = movm_t(pack_bf16(p[2], p[3]));   // keys 16 mt + 8..15
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 4);
                    psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 8);
                    psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 16);
                    lrun[h] = lrun[h] * corr[h] + psum[h];
                }
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    o[mt][0] *= corr[0];
                    o[mt][1] *= corr[1];
                    o[mt][2] *= corr[0];
                    o[mt][3] *= corr[1];
                }
                // ---- O^T += V^T P^T ----
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {        // dims 16 mt .. + 15
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {    // keys 16 kst .. + 15 of this warp's half
                        const int kst = 2 * hf + k2;
                        // matrices (transposed on load): (keys +0..7, dims +0..7), (keys +0..7, dims +8..15),
                        // (keys +8..15, dims +0..7), (keys +8..15, dims +8..15)
                        const int key = 16 * kst + (lane & 7) + (lane >> 4) * 8;
                        const int chunk = 2 * mt + ((lane >> 3) & 1);
                        const uint32_t addr = sw_addr(chunk < 8 ? vb0 : vb1, key, chunk & 7);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_t(addr, a0, a1, a2, a3);
                        mma_bf16(o[mt], a0, a1, a2, a3, pb[k2][0], pb[k2][1]);
                    }
                }
            }
            tc::fence_async_shared();   // zeroed rows are rewritten by TMA next
            __syncwarp();
            // a stage is handed back only once its copy has landed: after a wait
            // gave up, the producer never reuses a stage with a copy in flight
            if (ok && lane == 0) tc::mbar_arrive(&empty[s]);
        }

        // ---- every consumer warp publishes its (m, l, O^T); a failed warp
        // publishes l = NaN, which reaches every output it touches ----
        {
            float* x = xch + cw * kXchF;
            if (gq == 0) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    x[2 * tq + h] = mrun[h];
                    x[8 + 2 * tq + h] = ok ? lrun[h] : __int_as_float(0x7fc00000);
                }
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int dim = 16 * mt + gq + (e >> 1) * 8, h = 2 * tq + (e & 1);
                    x[16 + h * kXchRow + dim] = o[mt][e];
                }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsWarps) : "memory");
        const int t = threadIdx.x - 32;                 // 0 .. 32 kConsWarps - 1
        const bool bad = *abort != 0;
        // The CTA's own merge of the six states for (head h, dims 4 q4 .. 4 q4 + 3):
        //   m = max_w m_w,  l = sum_w 2^(m_w - m) l_w,  O = sum_w 2^(m_w - m) O_w
        auto local_merge = [&](int h, int q4, float& m, float& l, float4& ov) {
            m = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsWarps; ++w) m = fmaxf(m, xch[w * kXchF + h]);
            l = 0.f;
            ov = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kConsWarps; ++w) {
                const float* x = xch + w * kXchF;
                const float mw = x[h];
                const float wt = mw == -INFINITY ? 0.f : exp2f(mw - m);
                l = fmaf(wt, x[8 + h], l);
                const float4 ow = reinterpret_cast<const float4*>(x + 16 + h * kXchRow)[q4];
                ov.x = fmaf(wt, ow.x, ov.x);
                ov.y = fmaf(wt, ow.y, ov.y);
                ov.z = fmaf(wt, ow.z, ov.z);
                ov.w = fmaf(wt, ow.w, ov.w);
            }
        };
        __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.o) + ((int64_t)b * sh.Hq + (int64_t)g * G) * D;
        auto store_out = [&](int h, int q4, float4 ov, float l) {
            const float inv = 1.f / l;
            const bool nan = bad || !(l > 0.f);
            const float f = __int_as_float(0x7fc00000);
            reinterpret_cast<uint2*>(ob + (int64_t)h * D)[q4] =
                nan ? make_uint2(pack_bf16(f, f), pack_bf16(f, f))
                    : make_uint2(pack_bf16(ov.x * inv, ov.y * inv), pack_bf16(ov.z * inv, ov.w * inv));
        };
        if constexpr (kClu) {
            const int cs = a.cs;
            if (cs == 1) {
                for (int e = t; e < G * (D / 4); e += 32 * kConsWarps) {
                    const int h = e / (D / 4), q4 = e - h * (D / 4);
                    float m, l;
                    float4 ov;
                    local_merge(h, q4, m, l, ov);
                    store_out(h, q4, ov, l);
                }
            } else {
                // the leader's receive buffer: [cs - 1][G][kRecF] floats
                const uint32_t recv_off = cs == 2 ? L::kMerge : (uint32_t)kCons * kItemBytes;
                if (rank != 0) {
                    // store this CTA's partial into the leader once its barriers exist
                    cluster_wait();
                    const uint32_t dst = map_shared(sbase + recv_off, 0u) + ((rank - 1) * G * kRecF) * 4u;
                    const uint32_t rbar = map_shared(smem_u32(rcv), 0u);
                    for (int e = t; e < G * (D / 4); e += 32 * kConsWarps) {
                        const int h = e / (D / 4), q4 = e - h * (D / 4);
                        float m, l;
                        float4 ov;
                        local_merge(h, q4, m, l, ov);
                        if (bad) l = __int_as_float(0x7fc00000);
                        st_async_f32x4(dst + (uint32_t)(h * kRecF + 4 * q4) * 4u, ov, rbar);
                        if (q4 == 0) st_async_f32x4(dst + (uint32_t)(h * kRecF + D) * 4u, make_float4(m, l, 0.f, 0.f), rbar);
                    }
                } else {
                    // the CTA's own merge first, while the other partials are on their way
                    constexpr int kPer = (8 * (D / 4) + 32 * kConsWarps - 1) / (32 * kConsWarps);
                    float lm[kPer], ll[kPer];
                    float4 lo[kPer];
#pragma unroll
                    for (int k = 0; k < kPer; ++k) {
                        const int e = t + k * 32 * kConsWarps;
                        if (e < G * (D / 4)) local_merge(e / (D / 4), e % (D / 4), lm[k], ll[k], lo[k]);
                    }
                    // A sender that gave up on a wait still stores (NaN) within
                    // about one wait limit plus its own few microseconds of work:
                    // wait three limits, and never less than 10 ms, before giving
                    // up here -- a store into the shared memory of a leader that
                    // has already exited must not happen.
                    const unsigned long long lim = 3ull * g_sas_wait_limit_ns;
                    const bool got = rcv_wait(rcv, lim > kRecvFloorNs ? lim : kRecvFloorNs);
                    if (!got && t == 0) atomicAdd(&g_sas_wait_timeouts, 1u);
                    const float* rv = reinterpret_cast<const float*>(sm + recv_off);
#pragma unroll
                    for (int k = 0; k < kPer; ++k) {
                        const int e = t + k * 32 * kConsWarps;
                        if (e >= G * (D / 4)) break;
                        const int h = e / (D / 4), q4 = e - h * (D / 4);
                        const float m = lm[k], l = ll[k];
                        const float4 ov = lo[k];
                        float M = m;
                        for (int r = 0; r < cs - 1; ++r) M = fmaxf(M, rv[(r * G + h) * kRecF + D]);
                        const float w0 = m == -INFINITY ? 0.f : exp2f(m - M);
                        float Ls = w0 * l;
                        float4 acc = make_float4(w0 * ov.x, w0 * ov.y, w0 * ov.z, w0 * ov.w);
                        for (int r = 0; r < cs - 1; ++r) {
                            const float* x = rv + (r * G + h) * kRecF;
                            const float mr = x[D];
                            const float wr = mr == -INFINITY ? 0.f : exp2f(mr - M);
                            Ls = fmaf(wr, x[D + 1], Ls);
                            const float4 v = reinterpret_cast<const float4*>(x)[q4];
                            acc.x = fmaf(wr, v.x, acc.x);
                            acc.y = fmaf(wr, v.y, acc.y);
                            acc.z = fmaf(wr, v.z, acc.z);
                            acc.w = fmaf(wr, v.w, acc.w);
                        }
                        if (!got) Ls = __int_as_float(0x7fc00000);
                        store_out(h, q4, acc, Ls);
                    }
                }
            }
        } else {
            // the CTA's record of group bg: O, m, l of each head, 16-byte rows
            float* rec = a.part + (cta + bg) * (int64_t)G * kRecF;
            for (int e = t; e < G * (D / 4); e += 32 * kConsWarps) {
                const int h = e / (D / 4), q4 = e - h * (D / 4);
                float m, l;
                float4 ov;
                local_merge(h, q4, m, l, ov);
                if (bad) l = __int_as_float(0x7fc00000);
                reinterpret_cast<float4*>(rec + h * kRecF)[q4] = ov;
                if (q4 == 0) { rec[h * kRecF + D] = m; rec[h * kRecF + D + 1] = l; }
            }
            // the last CTA of the group to get here merges its records
            __threadfence();
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsWarps) : "memory");   // xch is free
            if (t == 0) {
                const int64_t c_first = flat_owner(fp, bg * nblk), c_last = flat_owner(fp, (bg + 1) * nblk - 1);
                *s_last = atomicAdd(&a.fin[bg], 1) == (int)(c_last - c_first);
            }
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsWarps) : "memory");   // s_last is set
            if (*s_last) {
                // Both consumer warps merge the group's records:
                //   o = sum_r 2^(m_r - M) O_r / sum_r 2^(m_r - M) l_r,  M = max_r m_r,
                // staging every record's (m, l) first so that all loads are in flight together.
                __threadfence();
                const int64_t c_first = flat_owner(fp, bg * nblk), c_last = flat_owner(fp, (bg + 1) * nblk - 1);
                const int R = (int)(c_last - c_first + 1);      // <= kMaxRecs by the plan
                const float* base = a.part + (c_first + bg) * (int64_t)G * kRecF;   // records are consecutive
                for (int e = t; e < R * G; e += 32 * kConsWarps) {
                    s_mg[e] = __ldcg(base + (int64_t)e * kRecF + D);
                    s_lg2[e] = __ldcg(base + (int64_t)e * kRecF + D + 1);
                }
                asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsWarps) : "memory");
                if (t < G) {
                    float M = -INFINITY, Lsum = 0.f;
                    for (int r = 0; r < R; ++r) M = fmaxf(M, s_mg[r * G + t]);
                    for (int r = 0; r < R; ++r) {
                        const float mr = s_mg[r * G + t];
                        const float w = mr == -INFINITY ? 0.f : exp2f(mr - M);
                        s_wg[r * G + t] = w;
                        Lsum = fmaf(w, s_lg2[r * G + t], Lsum);
                    }
                    const float inv = 1.f / Lsum;
                    for (int r = 0; r < R; ++r) s_wg[r * G + t] *= inv;
                }
                asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsWarps) : "memory");
                for (int e = t; e < G * (D / 4); e += 32 * kConsWarps) {
                    const int h = e / (D / 4), q4 = e - h * (D / 4);
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
                    for (int r = 0; r < R; ++r) {
                        const float w = s_wg[r * G + h];
                        const float4 v = __ldcg(reinterpret_cast<const float4*>(base + ((int64_t)r * G + h) * kRecF) + q4);
                        acc.x = fmaf(w, v.x, acc.x);
                        acc.y = fmaf(w, v.y, acc.y);
                        acc.z = fmaf(w, v.z, acc.z);
                        acc.w = fmaf(w, v.w, acc.w);
                    }
                    reinterpret_cast<uint2*>(ob + (int64_t)h * D)[q4] =
                        make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
                }
                // s_mg .. s_wg are read again only after the next segment's barriers
            }
        }
        seg = seg_end;
    }
}

// Merge the splits of one (b, kv head, query head):
//   o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
// The split weights are formed once in shared memory; each thread then reads
// its output column of every split with independent loads.
constexpr int kMaxSplits = 1024;

template <typename T, int D>
__global__ void __launch_bounds__(128)
decode_combine_kernel(Shape sh, const float* __restrict__ part, int splits, T* __restrict__ o) {
    __shared__ float w[kMaxSplits];
    __shared__ float red[4];
    const int G = sh.G;
    const int h = blockIdx.x % G;
    const int64_t bg = blockIdx.x / G;
    const int b = (int)(bg / sh.Hkv), g = (int)(bg % sh.Hkv);
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    auto rec = [&](int s) { return part + ((bg * splits + s) * G + h) * (int64_t)(D + 2); };
    float m = -INFINITY;
    for (int s = tid; s < splits; s += 128) m = fmaxf(m, rec(s)[D]);
    m = warp_max(m);
    if (lane == 0) red[wp] = m;
    __syncthreads();
    const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    float l = 0.f;
    for (int s = tid; s < splits; s += 128) {
        const float* r = rec(s);
        const float ws = r[D] == -INFINITY ? 0.f : exp2f(r[D] - M);
        w[s] = ws;
        l = fmaf(ws, r[D + 1], l);
    }
    l = warp_sum(l);
    if (lane == 0) red[wp] = l;
    __syncthreads();
    const float L = red[0] + red[1] + red[2] + red[3];
    for (int d = tid; d < D; d += 128) {
        float acc = 0.f;
#pragma unroll 8
        for (int s = 0; s < splits; ++s) acc = fmaf(w[s], rec(s)[d], acc);
        o[((int64_t)b * sh.Hq + (int64_t)g * G + h) * D + d] = Elem<T>::from_f(acc / L);
    }
}

template <typename T, int D, int GMAX, int BS>
cudaError_t run_decode(const DecArgs& a, cudaStream_t st) {
    constexpr size_t smem = dec_smem_bytes<T, D, GMAX, BS>();
    auto kern = decode_partial_kernel<T, D, GMAX, BS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)a.sh.B * a.sh.Hkv * a.splits;
    {
        KernelTimer kt("decode_partial", st);
        kern<<<(unsigned)grid, kDecThreads, smem, st>>>(a);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    {
        KernelTimer kt("decode_combine", st);
        decode_combine_kernel<T, D><<<(unsigned)(a.sh.B * a.sh.Hkv * a.sh.G), 128, 0, st>>>(a.sh, a.part, a.splits,
                                                                                           static_cast<T*>(a.o));
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

// SMs of the current device (148 on B200), bounded by kMaxDecodeCtas; 148 if
// the query fails.
int decode_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess || n <= 0)
        n = 148;
    return std::min(n, kMaxDecodeCtas);
}

constexpr size_t kFlatSmemBytes = FlatSmem::kTotal + 1024;

// Clusters of cs CTAs that the current device can hold at once (0 if the
// query fails), looked up once per device and size.
int max_active_clusters(int cs) {
    constexpr int kDevs = 64;
    static std::mutex mu;
    static int cache[kDevs][kMaxCluster + 1];
    static bool known[kDevs][kMaxCluster + 1];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevs || cs < 1 || cs > kMaxCluster) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!known[dev][cs]) {
        int n = 0;
        if (cudaFuncSetAttribute(decode_flat_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kFlatSmemBytes) == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)cs);
            cfg.blockDim = dim3(kFlatThreads);
            cfg.dynamicSmemBytes = kFlatSmemBytes;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)cs;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, decode_flat_kernel<true>, &cfg) != cudaSuccess) n = 0;
        }
        (void)cudaGetLastError();
        cache[dev][cs] = n;
        known[dev][cs] = true;
    }
    return cache[dev][cs];
}

// Cluster size of the tensor-core decode, 0 for the flat split. Short block
// lists (a sparse selection: nblk <= 128) with at most one group per SM get
// one cluster per group, as large as every cluster stays resident at once
// (<= 8, <= nblk, groups x cs <= SMs): the partials then meet in the leader's
// shared memory, and no record, counter or second pass over L2 is needed.
// Long lists (dense decode) and more groups than SMs use the flat split.
int decode_cluster_size(int64_t groups, int nblk) {
    if (nblk > 128 || groups > decode_sms()) return 0;
    for (int cs = kMaxCluster; cs >= 1; cs >>= 1)
        if (cs <= nblk && groups * cs <= decode_sms() && (cs == 1 || max_active_clusters(cs) >= groups)) return cs;
    return 0;
}

cudaError_t run_decode_flat(DecArgs a, cudaStream_t st) {
    CUtensorMap mk, mv;
    const uint64_t rows = a.table == nullptr ? (uint64_t)a.sh.B * a.sh.Hkvp * (uint64_t)a.stride
                                             : (uint64_t)a.num_pages * a.sh.Hkvp * 64;
    if (!encode_bf16_2d(&mk, a.kc, rows, 128, 64) || !encode_bf16_2d(&mv, a.vc, rows, 128, 64))
        return cudaErrorInvalidValue;
    const int64_t groups = (int64_t)a.sh.B * a.sh.Hkv;
    a.cs = decode_cluster_size(groups, a.fp.nblk);
    cudaError_t e;
    if (a.cs > 0) {
        e = cudaFuncSetAttribute(decode_flat_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kFlatSmemBytes);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(groups * a.cs));
        cfg.blockDim = dim3(kFlatThreads);
        cfg.dynamicSmemBytes = kFlatSmemBytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)a.cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        {
            KernelTimer kt("decode_flat", st);
            e = cudaLaunchKernelEx(&cfg, decode_flat_kernel<true>, mk, mv, a);
        }
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e == cudaSuccess) count_launches(1);
        return e;
    }
    e = cudaFuncSetAttribute(decode_flat_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kFlatSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(a.fin, 0, sizeof(int) * (size_t)groups, st);
    if (e != cudaSuccess) return e;
    {
        KernelTimer kt("decode_flat", st);
        decode_flat_kernel<false><<<(unsigned)a.fp.ncta, kFlatThreads, kFlatSmemBytes, st>>>(mk, mv, a);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

template <typename T, int D, int BS>
cudaError_t decode_g(const DecArgs& a, cudaStream_t st) {
    if (a.sh.G <= 4) return run_decode<T, D, 4, BS>(a, st);
    return run_decode<T, D, 8, BS>(a, st);
}
template <typename T, int D>
cudaError_t decode_b(const DecArgs& a, cudaStream_t st) {
    if (a.sh.bs == 32) return decode_g<T, D, 32>(a, st);
    return decode_g<T, D, 64>(a, st);
}
template <typename T>
cudaError_t decode_d(const DecArgs& a, cudaStream_t st) {
    if (a.sh.D == 64) return decode_b<T, 64>(a, st);
    return decode_b<T, 128>(a, st);
}

}  // namespace

// The tensor-core path (bf16, d 128, block 64, G <= 8) with TMA row
// coordinates that fit in int32.
static bool decode_flat_supported(const Shape& s, int64_t stride) {
    return s.dtype == SAS_DT_BF16 && s.D == 128 && s.bs == 64 && s.G <= 8 &&
           (int64_t)s.B * s.Hkvp * stride <= (int64_t)INT32_MAX;
}

static FlatPlan flat_plan(const Shape& s, bool dense) {
    const int64_t C = s.q_offset / s.bs;
    FlatPlan f;
    f.nblk = (int)(dense ? C + 1 : std::min<int64_t>(s.K, C) + 1);
    f.W = (int64_t)s.B * s.Hkv * f.nblk;
    // each CTA takes >= kCons items (one per consumer warp; few records per
    // group), and a group spans at most kMaxRecs CTAs:
    // ceil(nblk / per) + 1 <= kMaxRecs
    const int64_t min_per = std::max<int64_t>(kCons, (f.nblk + kMaxRecs - 3) / (kMaxRecs - 2));
    f.ncta = (int)std::max<int64_t>(1, std::min<int64_t>(decode_sms(), f.W / min_per));
    f.per = f.W / f.ncta;
    f.rem = f.W % f.ncta;
    return f;
}

// Records of the tensor-core path: at most one per (CTA, group it touches),
// i.e. ncta - 1 + groups, numbered c + bg; then the per-group counters.
static size_t flat_record_bytes(const Shape& s) {
    const size_t recs = (size_t)kMaxDecodeCtas + (size_t)s.B * s.Hkv;
    return (sizeof(float) * recs * s.G * kRecF + 255) & ~(size_t)255;
}

// CUDA-core path: `splits` CTAs of `bpc` blocks per (b, kv head), merged by a
// second kernel.
DecodePlan decode_plan(const Shape& s, bool dense) {
    DecodePlan p;
    const int64_t C = s.q_offset / s.bs;
    if (!dense) {
        p.bpc = 1;
        p.splits = s.K + 1;
        return p;
    }
    const int64_t nblk = C + 1;
    const int64_t groups = (int64_t)s.B * s.Hkv;
    const int64_t target = 148 * 3;   // CTAs: one wave (three ~67 KB, 256-thread CTAs fit per SM)
    int64_t bpc = (groups * nblk + target - 1) / target;
    bpc = std::max<int64_t>(bpc, (nblk + kMaxSplits - 1) / kMaxSplits);   // the merge takes <= kMaxSplits
    bpc = std::max<int64_t>(1, bpc);
    p.bpc = (int)bpc;
    p.splits = (int)((nblk + bpc - 1) / bpc);
    return p;
}

cudaError_t launch_decode(const Shape& s, const void* q, const void* kc, const void* vc, int64_t stride,
                          const int32_t* idx, const float* gl, const int32_t* nsel, void* o, float* part,
                          cudaStream_t st) {
    const bool dense = idx == nullptr;
    if (decode_flat_supported(s, stride)) {
        DecArgs a{s, q, kc, vc, stride, idx, gl, nsel, part, o, 0, 0, flat_plan(s, dense), nullptr, 0,
                  nullptr, 0, 0, nullptr};
        a.fin = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(part) + flat_record_bytes(s));
        return run_decode_flat(a, st);
    }
    const DecodePlan p = decode_plan(s, dense);
    DecArgs a{s, q, kc, vc, stride, idx, gl, nsel, part, o, p.bpc, p.splits, FlatPlan{}, nullptr, 0,
              nullptr, 0, 0, nullptr};
    if (s.dtype == SAS_DT_FP32) return decode_d<float>(a, st);
    return decode_d<__nv_bfloat16>(a, st);
}

cudaError_t set_decode_wait_limit(unsigned long long ns) {
    return cudaMemcpyToSymbol(g_sas_wait_limit_ns, &ns, sizeof(ns));
}

bool decode_paged_supported(const Shape& s, int64_t num_pages) {
    return s.dtype == SAS_DT_BF16 && s.D == 128 && s.bs == 64 && s.G <= 8 && num_pages >= 1 &&
           num_pages * s.Hkvp * 64 <= (int64_t)INT32_MAX;
}

cudaError_t launch_decode_paged(const Shape& s, const void* q, const void* kp, const void* vp, int num_pages,
                                const int32_t* table, int max_blocks, const int32_t* lens, const int32_t* idx,
                                const float* gl, const int32_t* nsel, void* o, float* part, cudaStream_t st) {
    const bool dense = idx == nullptr;
    DecArgs a{s, q, kp, vp, 0, idx, gl, nsel, part, o, 0, 0, flat_plan(s, dense), nullptr, 0,
              table, max_blocks, num_pages, lens};
    a.fin = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(part) + flat_record_bytes(s));
    return run_decode_flat(a, st);
}

cudaError_t read_decode_timeouts(unsigned int* out) {
    return cudaMemcpyFromSymbol(out, g_sas_wait_timeouts, sizeof(unsigned int));
}

size_t decode_ws_bytes(const Shape& s) {
    // covers both layouts (the cache stride, which picks the path, is not known here)
    const DecodePlan a = decode_plan(s, false), b = decode_plan(s, true);
    const int64_t splits = std::max(a.splits, b.splits);
    const size_t simt = sizeof(float) * (size_t)s.B * s.Hkv * splits * s.G * (s.D + 2);
    const size_t flat = flat_record_bytes(s) + sizeof(int) * (size_t)s.B * s.Hkv;
    return std::max(simt, flat);
}

}  // namespace sas

// ------------------------------------------------- decode without allocation ---
//
// Some callers of decode cannot call cudaMalloc at all: code that runs with a
// fixed memory budget carved out up front, plug-ins whose host framework owns
// every device allocation, or paths where an allocation (or its implicit
// synchronisation) is not allowed. For them, sas_sparse_decode_noalloc keeps the
// split partials in this file-scope device array instead of a caller workspace.
// Every GPU that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SAS_NOALLOC_SCRATCH_BYTES];

namespace sas {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
cudaError_t noalloc_scratch(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = static_cast<float*>(g_scratch_ptr[dev]);
    return cudaSuccess;
}

}  // namespace

}  // namespace sas

extern "C" sas_status sas_sparse_decode_noalloc(const sas_desc* desc, const void* q, const void* k_cache,
                                                const void* v_cache, int64_t cache_stride_tokens,
                                                const int32_t* idx, const float* gate_logit,
                                                const int32_t* n_sel, void* o, void* stream) {
    using namespace sas;
    Shape s;
    sas_status st = check_decode_args(desc, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o, &s);
    if (st != SAS_OK) return st;
    if (decode_ws_bytes(s) > (size_t)SAS_NOALLOC_SCRATCH_BYTES) return SAS_ERR_WORKSPACE;
    float* part = nullptr;
    if (noalloc_scratch(&part) != cudaSuccess) return SAS_ERR_CUDA;
    // Every split record is written before the merge reads it; the per-group
    // counters that pick the merging CTA are zeroed by the call itself.
    const cudaError_t e = launch_decode(s, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o,
                                        part, (cudaStream_t)stream);
    return e == cudaSuccess ? SAS_OK : SAS_ERR_CUDA;
}
