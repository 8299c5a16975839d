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
// of every later query tile and writes the block's own 64 tokens. Then a
// group of lanes per row places the row's kept (row, slot) entries: the position of token t in
// block j's run is the count before t's tile plus the set bits of the tile's
// bitmap word below t -- no search. Entry e:
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

// kL lanes per (b, g, t) row (16 when K <= 16, two rows per warp, else 32):
// they load the row's per-head values, kept blocks and log-gates together and
// broadcast the values to the group, then each kept slot (one lane each)
// places its entry and the row values (rvs <= 16 floats, 16-byte stores) in
// an earlier block's run.
template <int kL>
__global__ void __launch_bounds__(kThreads)
sel_stream_fill_kernel(Shape sh, const uint64_t* __restrict__ maskT, const int32_t* __restrict__ idx,
                       const float* __restrict__ gl, const int32_t* __restrict__ nsel, const float* __restrict__ v0,
                       const float* __restrict__ v1, int vals, SelStream st) {
    const int sub = (threadIdx.x & 31) / kL, li = threadIdx.x & (kL - 1);
    const int64_t row = ((int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5)) * (32 / kL) + sub;
    const bool ok = row < sh.rows();               // no early exit: the groups shuffle
    const int bg = ok ? (int)(row / sh.T) : 0;
    const int t = ok ? (int)(row - (int64_t)bg * sh.T) : 0;
    const int tau = t / kBS;
    const int b = bg / sh.Hkv, g = bg - b * sh.Hkv;
    const int nv = sh.G * vals;                    // <= 16
    float myv = 0.f;
    if (ok && li < nv) {
        const int h = li / vals, v = li - h * vals;
        const int64_t qrow = ((int64_t)b * sh.Hq + g * sh.G + h) * sh.T + t;
        myv = v == 0 ? v0[qrow] : v1[qrow];
    }
    const int ns = ok ? nsel[row] : 0;
    const uint64_t below = (1ull << (t & (kBS - 1))) - 1ull;
    for (int s0 = 0; s0 < sh.K; s0 += kL) {         // uniform across the warp
        const int slot = s0 + li;
        int j = -1;
        float lg = 0.f;
        if (ok && slot < sh.K) {
            j = idx[row * sh.K + slot];
            lg = gl[row * sh.K + slot];
        }
        float rowv[kMaxRvs];
#pragma unroll
        for (int v = 0; v < kMaxRvs; ++v) rowv[v] = __shfl_sync(0xffffffffu, myv, v, kL);   // 0 past G * vals
        // the own block is written by the index kernel
        if (slot < ns && j >= 0 && j < tau) {
            const int64_t blk = (int64_t)bg * sh.NB + j;
            const int64_t pos = (int64_t)st.base[blk] + st.pre[blk * sh.nT + tau] +
                                __popcll(maskT[blk * sh.nT + tau] & below);
            st.ent[pos] = make_int4(t, __float_as_int(lg), slot, 0);
            float4* out = reinterpret_cast<float4*>(st.rv + pos * st.rvs);
#pragma unroll
            for (int v = 0; v < kMaxRvs; v += 4)
                if (v < st.rvs) out[v / 4] = make_float4(rowv[v], rowv[v + 1], rowv[v + 2], rowv[v + 3]);
        }
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
        KernelTimer kt("sel_stream_fill", stream);
        if (s.K <= 16) {
            const int64_t rpb = 2 * (kThreads / 32);
            sel_stream_fill_kernel<16><<<(unsigned)((s.rows() + rpb - 1) / rpb), kThreads, 0, stream>>>(
                s, maskT, idx, gl, nsel, v0, v1, vals, st);
        } else {
            const int64_t rpb = kThreads / 32;
            sel_stream_fill_kernel<32><<<(unsigned)((s.rows() + rpb - 1) / rpb), kThreads, 0, stream>>>(
                s, maskT, idx, gl, nsel, v0, v1, vals, st);
        }
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

}  // namespace sas
