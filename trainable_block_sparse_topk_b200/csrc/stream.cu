// stream.cu -- per-key-block token streams for the gathered-row tensor-core
// kernels.
//
// The gathered-row forward and backward give one CTA to each (key block j,
// batch, KV group) and walk the (token, head) rows whose attention includes
// block j: the block's own 64 tokens (causal current block), then every later
// token whose selection kept j (SAS study note 1-2 TopK, 2-2 gated attention;
// arXiv text 3 selected token set). This kernel lays that walk out once per
// call, so the attention kernels read it with contiguous bulk copies instead
// of searching the bitmap and the kept lists inside their pipelines.
//
// Two kernels build the streams. Per (j, b, g) one CTA counts the block's
// tokens from the column bitmap maskT[b,g,j,:], reserves a contiguous run of
// entries with one atomic add (runs of different blocks land in any order;
// each run's own order is fixed), stores the running token count at the start
// of every later query tile and writes the block's own 64 tokens. Then one
// CTA per query tile places the tile's kept (row, slot) entries, grouped by
// block: the position of token t in block j's run is the count before t's
// tile plus the set bits of the tile's bitmap word below t -- no search. Entry e:
//   ent[e] = {t, bits of log g_j(t), slot of j in t's ascending kept list, 0}
//            (log-gate 0 and slot -1 for the block's own tokens),
//   rv[e * rvs + h * vals + v] = row value v of query head h of token t.
#include "common.cuh"
#include "kernels.h"

namespace sas {

namespace {

constexpr int kBS = 64;
constexpr int kThreads = 256;
constexpr int kMaxRvs = 16;   // G <= 8 heads x 2 values

__device__ __forceinline__ void put_rows(const Shape& sh, int b, int g, int t, const float* __restrict__ v0,
                                         const float* __restrict__ v1, int vals, float* out) {
    for (int h = 0; h < sh.G; ++h) {
        const int64_t qrow = ((int64_t)b * sh.Hq + g * sh.G + h) * sh.T + t;
        out[h * vals] = v0[qrow];
        if (vals == 2) out[h * vals + 1] = v1[qrow];
    }
}

// One CTA per (j, b, g): count, reservation, per-tile running counts, own tokens.
__global__ void __launch_bounds__(kThreads)
sel_stream_index_kernel(Shape sh, const uint64_t* __restrict__ maskT, const float* __restrict__ v0,
                        const float* __restrict__ v1, int vals, SelStream st) {
    __shared__ int s_part[32];
    __shared__ int s_base;
    const int ngroups = sh.B * sh.Hkv;
    const int j = (int)(blockIdx.x / ngroups);
    const int bg = (int)(blockIdx.x % ngroups);
    const int b = bg / sh.Hkv, g = bg % sh.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t blk = (int64_t)bg * sh.NB + j;
    const uint64_t* col = maskT + blk * sh.nT;
    int* pre = st.pre + blk * sh.nT;
    // per-tile counts, scanned in chunks of kThreads tiles
    int run = kBS;
    for (int t0 = 0; t0 < sh.nT; t0 += kThreads) {
        const int tau = t0 + tid;
        const int c = (tau < sh.nT && tau > j) ? __popcll(col[tau]) : 0;
        int inc = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31) s_part[warp] = inc;
        __syncthreads();
        int wsum = 0, total = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            wsum += w < warp ? s_part[w] : 0;
            total += s_part[w];
        }
        if (tau < sh.nT) pre[tau] = run + wsum + inc - c;
        run += total;
        __syncthreads();
    }
    if (tid == 0) {
        s_base = atomicAdd(st.counter, run);
        st.base[blk] = s_base;
        st.count[blk] = run;
    }
    __syncthreads();
    const int base = s_base;
    if (tid < kBS) {
        const int t = j * kBS + tid;
        const int64_t e = (int64_t)base + tid;
        st.ent[e] = make_int4(t, 0, -1, 0);
        put_rows(sh, b, g, t, v0, v1, vals, st.rv + e * st.rvs);
    }
}

// One CTA per (b, g, query tile tau) places the tile's kept (row, slot)
// entries. The tile's kept blocks, log-gates and per-head row values are read
// once (contiguous rows); the entries are bucketed by block in shared memory
// (count, scan, scatter), and consecutive threads then write consecutive
// entries of one block's segment for this tile -- the tokens of tile tau that
// kept block j occupy positions base + pre[tau] .. + popcount(bitmap word) of
// block j's run, so the stores coalesce instead of scattering one row's K
// entries over K runs. Position of token t in its segment: the set bits of the
// tile's bitmap word below t (the same for any processing order).
__global__ void __launch_bounds__(kThreads)
sel_stream_tile_kernel(Shape sh, const uint64_t* __restrict__ maskT, const int32_t* __restrict__ idx,
                       const float* __restrict__ gl, const int32_t* __restrict__ nsel, const float* __restrict__ v0,
                       const float* __restrict__ v1, int vals, SelStream st) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int K = sh.K, tid = threadIdx.x;
    const int bg = (int)(blockIdx.x / sh.nT);
    const int tau = (int)(blockIdx.x - (int64_t)bg * sh.nT);
    if (tau == 0) return;                            // tile 0 has no earlier block
    const int b = bg / sh.Hkv, g = bg - b * sh.Hkv;
    const int ne = kBS * K;                          // (token, slot) pairs of the tile
    const int rvs = st.rvs;
    int* s_j = reinterpret_cast<int*>(smem);                 // [ne] kept block, -1 if not placed here
    float* s_lg = reinterpret_cast<float*>(s_j + ne);        // [ne] its log-gate
    float* s_rv = s_lg + ne;                                 // [kBS][rvs] row values of the tile's tokens
    int* s_cnt = reinterpret_cast<int*>(s_rv + kBS * rvs);   // [tau] entries per block, then cursors
    uint16_t* s_ord = reinterpret_cast<uint16_t*>(s_cnt + tau);   // [ne] entry ids grouped by block
    __shared__ int s_part[kThreads / 32];
    const int64_t row0 = (int64_t)bg * sh.T + (int64_t)tau * kBS;   // the tile's first (b, g, t) row
    for (int e = tid; e < ne; e += kThreads) {
        const int tl = e / K, slot = e - tl * K;
        const int64_t row = row0 + tl;
        int j = slot < nsel[row] ? idx[row * K + slot] : -1;
        if (j >= tau) j = -1;                        // the own block is written by the index kernel
        s_j[e] = j;
        s_lg[e] = gl[row * K + slot];
    }
    for (int i = tid; i < kBS * rvs; i += kThreads) {   // token fastest: contiguous loads per head
        const int tl = i % kBS, k = i / kBS;
        const int h = k / vals, v = k - h * vals;
        float x = 0.f;
        if (h < sh.G) {
            const int64_t qrow = ((int64_t)b * sh.Hq + g * sh.G + h) * sh.T + (int64_t)tau * kBS + tl;
            x = v == 0 ? v0[qrow] : v1[qrow];
        }
        s_rv[tl * rvs + k] = x;
    }
    for (int i = tid; i < tau; i += kThreads) s_cnt[i] = 0;
    __syncthreads();
    for (int e = tid; e < ne; e += kThreads)
        if (s_j[e] >= 0) atomicAdd(&s_cnt[s_j[e]], 1);
    __syncthreads();
    // exclusive scan of the per-block counts: thread tid owns blocks
    // [tid * per, (tid + 1) * per)
    const int per = (tau + kThreads - 1) / kThreads;
    int mine = 0;
    for (int i = tid * per; i < min(tau, (tid + 1) * per); ++i) mine += s_cnt[i];
    const int lane = tid & 31, warp = tid >> 5;
    int inc = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s_part[warp] = inc;
    __syncthreads();
    int off = inc - mine;
    for (int w = 0; w < warp; ++w) off += s_part[w];
    int total = 0;
    for (int w = 0; w < kThreads / 32; ++w) total += s_part[w];
    for (int i = tid * per; i < min(tau, (tid + 1) * per); ++i) {
        const int c = s_cnt[i];
        s_cnt[i] = off;                              // cursor: first slot of block i's bucket
        off += c;
    }
    __syncthreads();
    for (int e = tid; e < ne; e += kThreads) {
        const int j = s_j[e];
        if (j >= 0) s_ord[atomicAdd(&s_cnt[j], 1)] = (uint16_t)e;
    }
    __syncthreads();
    for (int p = tid; p < total; p += kThreads) {
        const int e = s_ord[p];
        const int tl = e / K, slot = e - tl * K;
        const int j = s_j[e];
        const int64_t blk = (int64_t)bg * sh.NB + j;
        const int64_t pos = (int64_t)st.base[blk] + st.pre[blk * sh.nT + tau] +
                            __popcll(maskT[blk * sh.nT + tau] & ((1ull << tl) - 1ull));
        st.ent[pos] = make_int4(tau * kBS + tl, __float_as_int(s_lg[e]), slot, 0);
        const float4* src = reinterpret_cast<const float4*>(s_rv + tl * rvs);
        float4* dst = reinterpret_cast<float4*>(st.rv + pos * rvs);
        for (int v = 0; v < rvs / 4; ++v) dst[v] = src[v];
    }
}

}  // namespace

int sel_stream_rvs(const Shape& s, int vals) { return (s.G * vals + 3) & ~3; }

int64_t sel_stream_capacity(const Shape& s) { return (int64_t)s.B * s.Hkv * s.T * (s.K + 1); }

static size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t sel_stream_bytes(const Shape& s, int vals) {
    const size_t cap = (size_t)sel_stream_capacity(s);
    const size_t nblk = (size_t)s.B * s.Hkv * s.NB;
    return a256(16 * cap) + a256(4 * cap * (size_t)sel_stream_rvs(s, vals)) + 2 * a256(4 * nblk) +
           a256(4 * nblk * (size_t)s.nT) + 256;
}

SelStream sel_stream_at(void* ws, const Shape& s, int vals) {
    const size_t cap = (size_t)sel_stream_capacity(s);
    const size_t nblk = (size_t)s.B * s.Hkv * s.NB;
    unsigned char* p = static_cast<unsigned char*>(ws);
    SelStream st;
    st.rvs = sel_stream_rvs(s, vals);
    st.ent = reinterpret_cast<int4*>(p);
    p += a256(16 * cap);
    st.rv = reinterpret_cast<float*>(p);
    p += a256(4 * cap * (size_t)st.rvs);
    st.base = reinterpret_cast<int*>(p);
    p += a256(4 * nblk);
    st.count = reinterpret_cast<int*>(p);
    p += a256(4 * nblk);
    st.pre = reinterpret_cast<int*>(p);
    p += a256(4 * nblk * (size_t)s.nT);
    st.counter = reinterpret_cast<int*>(p);
    return st;
}

cudaError_t launch_sel_stream(const Shape& s, const uint64_t* maskT, const int32_t* idx, const float* gl,
                              const int32_t* nsel, const float* v0, const float* v1, int vals, const SelStream& st,
                              cudaStream_t stream) {
    if (st.rvs > kMaxRvs || st.rvs % 4 != 0) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(st.counter, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)s.B * s.Hkv * s.NB;
    {
        KernelTimer kt("sel_stream_index", stream);
        sel_stream_index_kernel<<<(unsigned)grid, kThreads, 0, stream>>>(s, maskT, v0, v1, vals, st);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    {
        // kept (row, slot) entries of query tiles 1 .. nT - 1 (tile 0 has none)
        const size_t smem = (size_t)kBS * s.K * 8 + (size_t)kBS * st.rvs * 4 + (size_t)s.nT * 4 + (size_t)kBS * s.K * 2;
        if (smem > 40 * 1024) {   // beside the static scan array
            e = cudaFuncSetAttribute(sel_stream_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        KernelTimer kt("sel_stream_fill", stream);
        sel_stream_tile_kernel<<<(unsigned)((int64_t)s.B * s.Hkv * s.nT), kThreads, smem, stream>>>(
            s, maskT, idx, gl, nsel, v0, v1, vals, st);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

}  // namespace sas
