// topk.cu -- exact top-k of index scores per query.
//
// "DeepSeek V4: Towards Highly Efficient Million Token Context Intelligence"
// (papers.chlience.com reading note), section 7: the selected set is the
// entries whose index score is in Top-k(I_{t,:}).  Ties go to the lower
// entry index; the output lists the chosen indices in ascending order.
//
// One row (one query's scores) is split over a thread-block cluster of CL
// CTAs (CL = 1..16), each holding a slice of at most 32768 scores in shared
// memory as order-preserving 32-bit keys.  The exact key T of the k-th
// largest score is found by range refinement: the cluster first agrees on
// the smallest and largest key [lo, hi]; each pass then histograms the keys
// inside [lo, hi] into at most 2048 bins of width 2^s, the cluster barrier
// publishes the per-CTA histograms, every CTA sums all CL of them through
// distributed shared memory and narrows [lo, hi] to the bin holding the
// k-th key (the same decision everywhere).  Three passes reach a single
// key.  Bins are uniform in key space, which is close to logarithmic in the
// score, so the skewed score distribution spreads over many bins and the
// shared-memory atomics rarely collide.  The selection is every key > T
// plus the first `need` keys == T in index order; a warp-ballot ordered
// compaction writes the indices ascending, with per-warp and per-CTA offsets
// from block and cluster prefix sums.  Hardware cluster barriers order
// everything: no flag spinning.
#include <algorithm>

#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace hca {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int64_t kSliceMax = 32768;
constexpr int64_t kSlicePref = 16384;

// Larger key = larger score; +0 and -0 map to the same key.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// CL (CTAs per row) is a template parameter so that the loops over the
// cluster's ranks unroll and all remote shared-memory loads are in flight
// together.
template <int CL>
__global__ void __launch_bounds__(kThreads)
topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ q_pos, int64_t Nc_cap,
            int m, int k, int64_t slice, int32_t* __restrict__ idx, int32_t* __restrict__ count) {
    constexpr int BPC = kBins / CL;                    // bins each CTA reduces for the cluster
    constexpr int V4 = BPC / 4;                        // uint4 per reduced slice
    static_assert(V4 * CL <= kThreads, "one remote uint4 per thread");
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int64_t row = blockIdx.x / CL;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    extern __shared__ uint32_t keys[];                 // [slice]
    __shared__ __align__(16) uint32_t hist[2][kBins];  // local histogram per pass
    __shared__ __align__(16) uint32_t stg[kThreads * 4];   // remote slices being reduced
    __shared__ __align__(16) uint32_t red[2][BPC];     // this CTA's reduced slice, published
    __shared__ uint32_t red_sum[2];                    // its total, published
    __shared__ __align__(8) uint32_t mm[2];            // published: slice min / max key
    __shared__ int pub[2];                             // published: ties, selected
    __shared__ uint32_t w_lo[kWarps], w_hi[kWarps];
    __shared__ int w_ties[kWarps], w_sel[kWarps];
    __shared__ int bc[4];

    int64_t E = (static_cast<int64_t>(q_pos[row]) + 1) / m;
    E = E < 0 ? 0 : (E > Nc_cap ? Nc_cap : E);
    const int K = static_cast<int>(E < k ? E : k);
    const bool take_all = (K == E);
    const int64_t lo_i = static_cast<int64_t>(rank) * slice;
    const int64_t hi_i = lo_i + slice < E ? lo_i + slice : E;
    const int n = hi_i > lo_i ? static_cast<int>(hi_i - lo_i) : 0;

    const float* src = scores + row * Nc_cap + lo_i;
    uint32_t tmin = 0xFFFFFFFFu, tmax = 0u;
    constexpr int kLd = 8;                               // loads in flight per thread
    for (int i0 = 0; i0 < n; i0 += kThreads * kLd) {
        float v[kLd];
#pragma unroll
        for (int u = 0; u < kLd; ++u) {
            const int i = i0 + u * kThreads + tid;
            v[u] = i < n ? __ldg(src + i) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kLd; ++u) {
            const int i = i0 + u * kThreads + tid;
            if (i < n) {
                const uint32_t kk = order_key(v[u]);
                keys[i] = kk;
                tmin = min(tmin, kk);
                tmax = max(tmax, kk);
            }
        }
    }
    uint32_t T = 0;
    int need = 0;
    if (!take_all) {
        // ---- cluster-wide key range: warp 0 lanes read one rank each
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            tmin = min(tmin, __shfl_xor_sync(0xffffffffu, tmin, o));
            tmax = max(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        }
        if (lane == 0) { w_lo[warp] = tmin; w_hi[warp] = tmax; }
        __syncthreads();
        if (tid == 0) {
            uint32_t a = 0xFFFFFFFFu, b = 0u;
            for (int w2 = 0; w2 < kWarps; ++w2) { a = min(a, w_lo[w2]); b = max(b, w_hi[w2]); }
            mm[0] = a; mm[1] = b;
        }
        cluster.sync();
        if (warp == 0) {
            uint32_t a = 0xFFFFFFFFu, b = 0u;
            if (lane < CL) {
                const uint2 rv = *reinterpret_cast<const uint2*>(cluster.map_shared_rank(mm, lane));
                a = rv.x; b = rv.y;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
                b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
            }
            if (lane == 0) { bc[2] = static_cast<int>(a); bc[3] = static_cast<int>(b); }
        }
        __syncthreads();
        uint32_t lo = static_cast<uint32_t>(bc[2]), hi = static_cast<uint32_t>(bc[3]);
        need = K;
        // ---- range refinement (at most 3 passes of <= 2048 bins)
        int pass = 0;
#pragma unroll 1
        while (lo < hi) {
            int sh = 0;
            while (((hi - lo) >> sh) >= static_cast<uint32_t>(kBins)) ++sh;
            const int pb = pass & 1;
            uint32_t* h = hist[pb];
            for (int i = tid; i < kBins; i += kThreads) h[i] = 0;
            __syncthreads();
            for (int i = tid; i < n; i += kThreads) {
                const uint32_t kk = keys[i];
                if (kk >= lo && kk <= hi) atomicAdd(&h[(kk - lo) >> sh], 1u);
            }
            cluster.sync();
            // reduce bins [rank*BPC, (rank+1)*BPC) over the cluster: thread t reads
            // uint4 (t % V4) of that slice from rank t / V4
            if (tid < V4 * CL) {
                const int r = tid / V4, c = tid % V4;
                *reinterpret_cast<uint4*>(&stg[tid * 4]) =
                    *reinterpret_cast<const uint4*>(cluster.map_shared_rank(h, r) + rank * BPC + c * 4);
            }
            __syncthreads();
            if (tid < V4) {
                uint4 a = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int r = 0; r < CL; ++r) {
                    const uint4 b = *reinterpret_cast<const uint4*>(&stg[(r * V4 + tid) * 4]);
                    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
                }
                *reinterpret_cast<uint4*>(&red[pb][tid * 4]) = a;
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t t = 0;
                for (int i = lane; i < BPC; i += 32) t += red[pb][i];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
                if (lane == 0) red_sum[pb] = t;
            }
            cluster.sync();
            // warp 0: which rank's slice holds the need-th largest, then which bin
            if (warp == 0) {
                int sr = 0;
                if (lane < CL) sr = static_cast<int>(*cluster.map_shared_rank(&red_sum[pb], lane));
                int v = sr;                                    // inclusive suffix sum over ranks >= lane
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_down_sync(0xffffffffu, v, o);
                    if (lane + o < 32) v += u;
                }
                const int above_r = v - sr;
                const bool hit = lane < CL && above_r < need && above_r + sr >= need;
                const uint32_t hm = __ballot_sync(0xffffffffu, hit);
                const int rs = __ffs(hm) - 1;
                const int above0 = __shfl_sync(0xffffffffu, above_r, rs);
                const uint32_t* sl = cluster.map_shared_rank(&red[pb][0], rs);
                // lane l owns bins [l * BPC/32, (l+1) * BPC/32) of that slice
                constexpr int PER = BPC / 32;
                uint32_t cnt[PER];
                int mine = 0;
#pragma unroll
                for (int j = 0; j < PER; ++j) { cnt[j] = sl[lane * PER + j]; mine += static_cast<int>(cnt[j]); }
                int w2 = mine;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_down_sync(0xffffffffu, w2, o);
                    if (lane + o < 32) w2 += u;
                }
                int acc = above0 + w2 - mine;
#pragma unroll
                for (int j = PER - 1; j >= 0; --j) {
                    const int cj = static_cast<int>(cnt[j]);
                    if (acc < need && acc + cj >= need) { bc[0] = rs * BPC + lane * PER + j; bc[1] = acc; }
                    acc += cj;
                }
            }
            __syncthreads();
            const uint64_t nlo = static_cast<uint64_t>(lo) + (static_cast<uint64_t>(bc[0]) << sh);
            const uint64_t nhi = nlo + ((1ull << sh) - 1ull);
            need -= bc[1];
            lo = static_cast<uint32_t>(nlo);
            hi = nhi < hi ? static_cast<uint32_t>(nhi) : hi;
            ++pass;
            __syncthreads();
        }
        T = lo;
    }

    // ---- ordered selection: warp w owns a contiguous range of the slice
    const int per_w = (n + kWarps - 1) / kWarps;
    const int ws = min(n, warp * per_w), we = min(n, ws + per_w);
    int ties = 0, above = 0;
    if (!take_all) {
        for (int j = ws; j < we; j += 32) {
            const int i = j + lane;
            const uint32_t kk = i < we ? keys[i] : 0u;
            ties += __popc(__ballot_sync(0xffffffffu, i < we && kk == T));
            above += __popc(__ballot_sync(0xffffffffu, i < we && kk > T));
        }
    }
    if (lane == 0) w_ties[warp] = ties;
    __syncthreads();
    if (tid == 0) {
        int t = 0;
        for (int w2 = 0; w2 < kWarps; ++w2) t += w_ties[w2];
        pub[0] = t;
    }
    cluster.sync();
    if (warp == 0) {                                   // ties in lower-ranked CTAs
        int v = (lane < rank) ? *cluster.map_shared_rank(&pub[0], lane) : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) bc[2] = v;
    }
    __syncthreads();
    int tie_base = bc[2];
    for (int w2 = 0; w2 < warp; ++w2) tie_base += w_ties[w2];
    int take_ties = need - tie_base;
    take_ties = take_ties < 0 ? 0 : (take_ties > ties ? ties : take_ties);
    const int sel = take_all ? (we - ws) : (above + take_ties);
    if (lane == 0) w_sel[warp] = sel;
    __syncthreads();
    if (tid == 0) {
        int t = 0;
        for (int w2 = 0; w2 < kWarps; ++w2) t += w_sel[w2];
        pub[1] = t;
    }
    cluster.sync();
    if (warp == 0) {                                   // selections in lower-ranked CTAs
        int v = (lane < rank) ? *cluster.map_shared_rank(&pub[1], lane) : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) bc[3] = v;
    }
    __syncthreads();
    int out_pos = bc[3];
    for (int w2 = 0; w2 < warp; ++w2) out_pos += w_sel[w2];

    int32_t* orow = idx + row * k;
    int tie_rank = tie_base;
    const uint32_t lt = (1u << lane) - 1u;
    for (int j = ws; j < we; j += 32) {
        const int i = j + lane;
        const bool in = i < we;
        const uint32_t kk = in ? keys[i] : 0u;
        const bool is_tie = in && !take_all && kk == T;
        const uint32_t tb = __ballot_sync(0xffffffffu, is_tie);
        const bool take = in && (take_all || kk > T || (is_tie && tie_rank + __popc(tb & lt) < need));
        const uint32_t sb = __ballot_sync(0xffffffffu, take);
        if (take) orow[out_pos + __popc(sb & lt)] = static_cast<int32_t>(lo_i + i);
        out_pos += __popc(sb);
        tie_rank += __popc(tb);
    }
    if (rank == 0) {
        for (int j = K + tid; j < k; j += kThreads) orow[j] = -1;
        if (tid == 0) count[row] = K;
    }
    cluster.sync();   // no CTA leaves while a peer may still read its shared memory
}

int g_max_cluster = 0;   // largest cluster size this device schedules for topk_kernel

template <int CL>
cudaError_t launch_cl(int R, int64_t slice, const float* scores, const int32_t* q_pos, int64_t Nc_cap, int m, int k,
                      int32_t* idx, int32_t* count, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSliceMax * sizeof(uint32_t)));
    if (e == cudaSuccess && CL > 8)
        e = cudaFuncSetAttribute(topk_kernel<CL>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(static_cast<int64_t>(R) * CL));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(slice) * sizeof(uint32_t);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, topk_kernel<CL>, scores, q_pos, Nc_cap, m, k, slice, idx, count);
}

// ------------------------------------------------------------------ few long rows
// Used when there are few rows (decode: one per sequence) of many scores; no
// clusters (the kernels are described in namespace wide).  Workspace per row
// (256-byte aligned): the key histogram u32[2048] and a header u32[64] (keys
// above bin T1, candidates, CTAs done), cleared by a memset on the stream
// before every call; then the above keys' indices u32[kMaxK] and the
// candidates' composite keys u64[Nc_cap].
namespace wide {

// Few long rows (decode: one row per sequence).  The 11-bit key histogram of
// each row comes first (built by the indexer's epilogue in the fused decode
// call, or by hist_kernel); then one select_kernel launch:
//   every CTA reads the histogram, finds the threshold bin T1 (the highest
//   bin whose count from the top reaches k) and scans its chunk of the row
//   once: the indices of the keys above bin T1 (all selected, fewer than k of
//   them) and the composite keys of the keys in bin T1 (the candidates) are
//   staged per warp in shared memory and appended to the row's two lists, one
//   atomic claim per warp and list (the order inside a list is irrelevant);
//   the CTA that finishes last (a counter per row, behind a memory fence)
//   resolves the row: a radix select over the candidates' composite keys
//   (score key, then the complement of the index, so that every composite is
//   unique and equal scores rank the lower index first) finds the exact
//   threshold; the above keys and the selected candidates set their bits in a
//   shared-memory bitmap of the row, whose block-wide scan places every
//   selected index at its rank, i.e. in ascending order, without a sort.
// No CTA waits for another: the last one to arrive does the rest.
constexpr int kBins = 2048;
constexpr int kThreads = 256;              // hist_kernel
constexpr int kSelThreads = 512;           // select_kernel
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMaxIt = 64;                 // select: at most 64 x 512 scores per CTA
constexpr int kCandSmem = 4096;            // candidates resolved from shared memory (else from L2)
constexpr int kMaxK = 4096;
constexpr int kWpt = 16;                   // bitmap words per thread
constexpr int kSegWords = kSelThreads * kWpt;   // 8192 words = 262144 entries per bitmap segment
constexpr int kWBuf = 64;                  // per-warp staging entries per list
// dynamic shared memory of select_kernel: the candidates (resolve), one bitmap
// segment (resolve; the per-warp staging during the scan)
constexpr size_t kSelSmem = static_cast<size_t>(kCandSmem) * 8 + static_cast<size_t>(kSegWords) * 4;
static_assert(kSelWarps * kWBuf * 12 <= kSegWords * 4, "staging fits in the bitmap segment");

__host__ __device__ inline size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Layout {
    size_t clear_bytes;     // histogram + header, cleared before every call
    size_t above_off;       // u32 [kMaxK]: indices of the keys above bin T1
    size_t cand_off;        // u64 [Nc_cap]: composite keys of the candidates
    size_t row_bytes;       // per-row stride
};

__host__ __device__ inline Layout layout(int64_t Nc_cap) {
    Layout L;
    L.clear_bytes = static_cast<size_t>(kBins) * 4 + 256;
    L.above_off = L.clear_bytes;
    L.cand_off = L.above_off + static_cast<size_t>(kMaxK) * 4;
    L.row_bytes = L.cand_off + round256(static_cast<size_t>(Nc_cap) * 8);
    return L;
}

struct RowWs {
    uint32_t* hist;
    uint32_t* hdr;          // [0] keys above bin T1, [1] candidates, [2] CTAs done
    uint32_t* above;
    unsigned long long* cand;
};

__device__ __forceinline__ RowWs row_ws(uint8_t* ws, int64_t Nc_cap, int64_t r) {
    const Layout L = layout(Nc_cap);
    uint8_t* base = ws + static_cast<size_t>(r) * L.row_bytes;
    RowWs w;
    w.hist = reinterpret_cast<uint32_t*>(base);
    w.hdr = w.hist + kBins;
    w.above = reinterpret_cast<uint32_t*>(base + L.above_off);
    w.cand = reinterpret_cast<unsigned long long*>(base + L.cand_off);
    return w;
}

__device__ __forceinline__ int64_t n_eligible(const int32_t* q_pos, int64_t r, int m, int64_t Nc_cap) {
    const int64_t e = (static_cast<int64_t>(q_pos[r]) + 1) / m;
    return e < 0 ? 0 : (e > Nc_cap ? Nc_cap : e);
}

// Score of entry e as an fp32 value: an fp32 score, or a bf16 score (uint16
// bits; the note's BF16 index scores) widened exactly.
__device__ __forceinline__ float score_at(const float* row, int64_t e) { return row[e]; }
__device__ __forceinline__ float score_at(const uint16_t* row, int64_t e) {
    return __uint_as_float(static_cast<uint32_t>(row[e]) << 16);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
hist_kernel(const T* __restrict__ scores, const int32_t* __restrict__ q_pos, int64_t Nc_cap, int m,
            int64_t chunk, uint8_t* __restrict__ ws) {
    __shared__ uint32_t sh[kBins];
    const int64_t r = blockIdx.y;
    const int64_t n = n_eligible(q_pos, r, m, Nc_cap);
    const int64_t e0 = static_cast<int64_t>(blockIdx.x) * chunk;
    const int64_t e1 = min(e0 + chunk, n);
    if (e0 >= e1) return;
    for (int i = threadIdx.x; i < kBins; i += kThreads) sh[i] = 0;
    __syncthreads();
    const T* row = scores + static_cast<size_t>(r) * Nc_cap;
    // eight loads in flight per thread before the shared-memory atomics
    for (int64_t e = e0 + threadIdx.x; e < e1; e += kThreads * 8) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = e + j * kThreads < e1 ? score_at(row, e + j * kThreads) : 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (e + j * kThreads < e1) atomicAdd(&sh[order_key(v[j]) >> 21], 1u);
    }
    __syncthreads();
    RowWs w = row_ws(ws, Nc_cap, r);
    for (int i = threadIdx.x; i < kBins; i += kThreads)
        if (sh[i]) atomicAdd(&w.hist[i], sh[i]);
}

// block-wide inclusive scan of one value per thread (kSelThreads threads)
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* sh_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < kSelWarps ? sh_warp[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kSelWarps) sh_warp[lane] = s;
    }
    __syncthreads();
    const uint32_t r = (warp > 0 ? sh_warp[warp - 1] : 0u) + x;
    __syncthreads();
    return r;
}

// Digit of a histogram h of nb bins (2048 or 1024; the largest digit is nb-1)
// at which the count from the top reaches `need`.  Block-wide.  s_out[0] =
// the digit, s_out[1] = need minus the count strictly above it, s_out[2] =
// the count in it.  (An inconsistent histogram, whose total is below need,
// leaves digit 0, need and 0: wrong but in bounds.)
__device__ __forceinline__ void find_digit(const uint32_t* h, uint32_t nb, uint32_t need, uint32_t* sh_warp, uint32_t* s_out) {
    const int t = threadIdx.x;
    if (t == 0) { s_out[0] = 0u; s_out[1] = need; s_out[2] = 0u; }
    const uint32_t per = nb / kSelThreads;
    uint32_t c[4] = {0u, 0u, 0u, 0u}, tot = 0;
    for (uint32_t j = 0; j < per; ++j) { c[j] = h[nb - 1 - per * t - j]; tot += c[j]; }
    const uint32_t incl = block_incl_scan(tot, sh_warp);     // (syncs: s_out initialised before any write)
    const uint32_t before = incl - tot;
    if (before < need && incl >= need) {
        uint32_t acc = before;
        for (uint32_t j = 0; j < per; ++j) {
            if (acc + c[j] >= need) { s_out[0] = nb - 1 - per * t - j; s_out[1] = need - acc; s_out[2] = c[j]; break; }
            acc += c[j];
        }
    }
    __syncthreads();
}

// A full bitmap segment in shared memory: thread t's kWpt = 16 words (entries
// 512 t .. 512 t + 511 of the segment) sit in four 16-byte slots, rotated by
// t / 2 so that the eight lanes of a 16-byte access phase hit eight
// different bank groups.  (A shorter segment, at fewer words per thread,
// keeps its words in order.)
__device__ __forceinline__ uint32_t slot_of(uint32_t t, uint32_t j) { return 4 * t + ((j + (t >> 1)) & 3u); }
// shared-memory word index of segment word wd
__device__ __forceinline__ uint32_t word_at(uint32_t wd) {
    return 4 * slot_of(wd >> 4, (wd >> 2) & 3u) + (wd & 3u);
}

// Warp-uniform append of the lanes of mask (one value each) to a list: staged
// in the warp's shared buffer while it has room (count in *n), else claimed
// in the row's list at once.
template <typename V>
__device__ __forceinline__ void append(unsigned mask, V val, V* stage, uint32_t& n, uint32_t* counter, V* list,
                                       uint32_t cap) {
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    const uint32_t c = __popc(mask);
    if (n + c <= static_cast<uint32_t>(kWBuf)) {
        if ((mask >> lane) & 1u) stage[n + __popc(mask & lt)] = val;
        n += c;
    } else {
        uint32_t b = 0;
        if (lane == 0) b = atomicAdd(counter, c);
        b = __shfl_sync(0xffffffffu, b, 0);
        if ((mask >> lane) & 1u) {
            const uint32_t at = b + __popc(mask & lt);
            if (at < cap) list[at] = val;
        }
    }
}

// Flush a warp's staged entries: one claim, then coalesced stores.
template <typename V>
__device__ __forceinline__ void flush(const V* stage, uint32_t n, uint32_t* counter, V* list, uint32_t cap) {
    const int lane = threadIdx.x & 31;
    __syncwarp();
    uint32_t b = 0;
    if (lane == 0 && n) b = atomicAdd(counter, n);
    b = __shfl_sync(0xffffffffu, b, 0);
    for (uint32_t i = lane; i < n; i += 32)
        if (b + i < cap) list[b + i] = stage[i];
}

template <typename T>
__global__ void __launch_bounds__(kSelThreads, 1)
select_kernel(const T* __restrict__ scores, const int32_t* __restrict__ q_pos, int64_t Nc_cap, int m, int k,
              int64_t chunk, uint8_t* __restrict__ ws, int32_t* __restrict__ idx, int32_t* __restrict__ count) {
    extern __shared__ __align__(16) unsigned long long dyn[];
    unsigned long long* s_cand = dyn;                                          // [kCandSmem]
    uint32_t* s_bits = reinterpret_cast<uint32_t*>(dyn + kCandSmem);           // [kSegWords]
    __shared__ uint32_t s_hist[kBins];
    __shared__ uint32_t sh_warp[32];
    __shared__ uint32_t s_dig[4];
    __shared__ uint32_t s_tot;
    __shared__ int s_last;

    const int64_t r = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();                                    // the scores and histograms are complete
    const int64_t n = n_eligible(q_pos, r, m, Nc_cap);
    const uint32_t kk = static_cast<uint32_t>(min(static_cast<int64_t>(k), n));
    int32_t* orow = idx + static_cast<size_t>(r) * k;
    if (kk == 0) {
        if (blockIdx.x == 0) {
            if (tid == 0) count[r] = 0;
            for (int j = tid; j < k; j += kSelThreads) orow[j] = -1;
        }
        return;
    }
    RowWs w = row_ws(ws, Nc_cap, r);
    const T* row = scores + static_cast<size_t>(r) * Nc_cap;
    const int64_t e0 = static_cast<int64_t>(blockIdx.x) * chunk;
    const int64_t e1 = min(e0 + chunk, n);
    const int n_it = e1 > e0 ? static_cast<int>((e1 - e0 + kSelThreads - 1) / kSelThreads) : 0;
    constexpr int kBatch = 32;                             // loads in flight per thread
    // the chunk's first batch of scores does not depend on the threshold: its loads
    // fly while the histogram is read and searched
    float v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
        const int64_t e = e0 + static_cast<int64_t>(j) * kSelThreads + warp * 32 + lane;
        v[j] = (j < n_it && e < e1) ? score_at(row, e) : 0.0f;
    }
    // ---- threshold bin T1 from the row's histogram (the same in every CTA)
    {
        uint32_t hv[kBins / kSelThreads];                  // all loads in flight, then the stores
#pragma unroll
        for (int j = 0; j < kBins / kSelThreads; ++j) hv[j] = __ldcg(w.hist + tid + j * kSelThreads);
#pragma unroll
        for (int j = 0; j < kBins / kSelThreads; ++j) s_hist[tid + j * kSelThreads] = hv[j];
    }
    __syncthreads();
    find_digit(s_hist, kBins, kk, sh_warp, s_dig);
    const uint32_t t1 = s_dig[0];
    // ---- one pass over this CTA's chunk: the above keys' indices and the
    // candidates' composite keys, staged per warp, appended to the row's lists
    {
        uint32_t* s_wa = s_bits + warp * kWBuf;
        unsigned long long* s_wc = reinterpret_cast<unsigned long long*>(s_bits + kSelWarps * kWBuf) + warp * kWBuf;
        uint32_t na = 0, nc = 0;
        for (int it0 = 0; it0 < n_it; it0 += kBatch) {
            if (it0 > 0) {
#pragma unroll
                for (int j = 0; j < kBatch; ++j) {
                    const int64_t e = e0 + static_cast<int64_t>(it0 + j) * kSelThreads + warp * 32 + lane;
                    v[j] = (it0 + j < n_it && e < e1) ? score_at(row, e) : 0.0f;
                }
            }
            // lane j keeps the two ballot words of step it0 + j (small unrolled body)
            uint32_t my_a = 0u, my_c = 0u;
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                if (it0 + j >= n_it) break;
                const bool live = e0 + static_cast<int64_t>(it0 + j) * kSelThreads + warp * 32 + lane < e1;
                const uint32_t bin = order_key(v[j]) >> 21;
                const unsigned above = __ballot_sync(0xffffffffu, live && bin > t1);
                const unsigned in_t1 = __ballot_sync(0xffffffffu, live && bin == t1);
                if (lane == j) { my_a = above; my_c = in_t1; }
            }
            // the steps with keys to append (rare), one at a time; a candidate's score is
            // read again (an L1 hit: this lane loaded it above)
            unsigned todo = __ballot_sync(0xffffffffu, (my_a | my_c) != 0u);
#pragma unroll 1
            while (todo) {
                const int j = __ffs(todo) - 1;
                todo &= todo - 1u;
                const unsigned am = __shfl_sync(0xffffffffu, my_a, j), cm = __shfl_sync(0xffffffffu, my_c, j);
                const int64_t e = e0 + static_cast<int64_t>(it0 + j) * kSelThreads + warp * 32 + lane;
                if (am) append<uint32_t>(am, static_cast<uint32_t>(e), s_wa, na, w.hdr + 0, w.above, kMaxK);
                if (cm) {
                    const uint32_t key = ((cm >> lane) & 1u) ? order_key(score_at(row, e)) : 0u;
                    append<unsigned long long>(cm, (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(~e),
                                               s_wc, nc, w.hdr + 1, w.cand, static_cast<uint32_t>(Nc_cap));
                }
            }
        }
        flush<uint32_t>(s_wa, na, w.hdr + 0, w.above, kMaxK);
        flush<unsigned long long>(s_wc, nc, w.hdr + 1, w.cand, static_cast<uint32_t>(Nc_cap));
    }
    pdl_trigger();                                 // most CTAs end here: let the next kernel be scheduled
    // ---- the last CTA of the row resolves it.  The barrier orders every thread's
    // list stores before thread 0's fence, which (being cumulative) releases them
    // all before the count; the last CTA's thread 0 fences again before its
    // threads read the other CTAs' stores.
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const bool last = atomicAdd(&w.hdr[2], 1u) == gridDim.x - 1;
        if (last) __threadfence();
        s_last = last;
    }
    __syncthreads();
    if (!s_last) return;
    const uint32_t n_above = min(min(__ldcg(w.hdr + 0), kk), static_cast<uint32_t>(kMaxK));
    const uint32_t n_cand = min(__ldcg(w.hdr + 1), static_cast<uint32_t>(Nc_cap));
    const bool cached = n_cand <= static_cast<uint32_t>(kCandSmem);
    // the row's bitmap, in segments of at most kSegWords words; a segment of nws
    // words gives every thread wpt words, the least power of two with
    // wpt * kSelThreads >= nws (a short row still spreads over all threads)
    const size_t nw = static_cast<size_t>((n + 31) / 32);
    auto seg_wpt = [&](size_t seg) {
        const size_t nws = min(nw - seg, static_cast<size_t>(kSegWords));
        uint32_t x = 1;
        while (static_cast<size_t>(x) * kSelThreads < nws) x <<= 1;
        return x;
    };
    uint32_t wpt = seg_wpt(0);
    // the above indices stay in registers; cached candidates go to shared memory
    // (both lists in one round of loads); the first bitmap segment is cleared
    constexpr int kPer = kMaxK / kSelThreads;
    static_assert(kCandSmem / kSelThreads == kPer, "one round covers both lists");
    uint32_t av[kPer];
    {
        unsigned long long cv[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const uint32_t i = tid + j * kSelThreads;
            av[j] = i < n_above ? __ldcg(w.above + i) : 0u;
            cv[j] = (cached && i < n_cand) ? __ldcg(w.cand + i) : 0ull;
        }
        for (uint32_t j = 0; j < wpt; ++j) s_bits[tid + j * kSelThreads] = 0u;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const uint32_t i = tid + j * kSelThreads;
            if (cached && i < n_cand) s_cand[i] = cv[j];
        }
    }
    __syncthreads();
    // entry e sets its bit in the segment starting at word seg: segment word wd sits
    // at word_at(wd) at 16 words per thread, else at wd (thread t's words t wpt ..
    // t wpt + wpt - 1, in order)
    auto mark = [&](uint32_t e, size_t seg) {
        const uint32_t e_lo = static_cast<uint32_t>(seg * 32);
        const uint32_t wd = (e - e_lo) >> 5;
        if (e >= e_lo && wd < wpt * static_cast<uint32_t>(kSelThreads))
            atomicOr(&s_bits[wpt == static_cast<uint32_t>(kWpt) ? word_at(wd) : wd], 1u << (e & 31u));
    };
    // the above keys of the first segment set their bits beside the radix select
    // (which works on other shared words)
#pragma unroll
    for (int j = 0; j < kPer; ++j)
        if (tid + j * kSelThreads < n_above) mark(av[j], 0);
    auto cand = [&](uint32_t c) { return cached ? s_cand[c] : __ldcg(w.cand + c); };
    uint32_t need = kk - n_above;
    // threshold: candidates whose composite, on the bits fixed so far, is >= prefix
    unsigned long long prefix = 0ull, fmask = 0ull;
    if (need < n_cand) {
        prefix = static_cast<unsigned long long>(t1) << 53;
        fmask = 0xFFE0000000000000ull;
        // digits of the composite below the 11 bits of bin T1: 11, 10 (the rest of
        // the score key), then 11, 11, 10 (the complemented index)
#pragma unroll 1
        for (int ps = 0; ps < 5; ++ps) {
            const int width = (ps == 1 || ps == 4) ? 10 : 11;
            const int shift = ps == 0 ? 42 : ps == 1 ? 32 : ps == 2 ? 21 : ps == 3 ? 10 : 0;
            const uint32_t nb = 1u << width;
            for (uint32_t i = tid; i < nb; i += kSelThreads) s_hist[i] = 0u;
            __syncthreads();
            for (uint32_t c = tid; c < n_cand; c += kSelThreads) {
                const unsigned long long v = cand(c);
                if ((v & fmask) == prefix) atomicAdd(&s_hist[(v >> shift) & (nb - 1u)], 1u);
            }
            __syncthreads();
            find_digit(s_hist, nb, need, sh_warp, s_dig);
            prefix |= static_cast<unsigned long long>(s_dig[0]) << shift;
            fmask |= static_cast<unsigned long long>(nb - 1u) << shift;
            need = s_dig[1];
            const bool whole = s_dig[2] == need;            // every key of this digit is selected
            __syncthreads();
            if (whole) break;
        }
    }
    // ---- output, per bitmap segment: the selected candidates (and, past the first
    // segment, the above keys) set their bits; a block-wide scan gives every set
    // bit its rank, and each index is stored at its rank in the output row, i.e.
    // in ascending order
    uint32_t written = 0;
    for (size_t seg = 0; seg < nw; seg += kSegWords) {
        if (seg > 0) {
            wpt = seg_wpt(seg);
            for (uint32_t j = 0; j < wpt; ++j) s_bits[tid + j * kSelThreads] = 0u;
            __syncthreads();
#pragma unroll
            for (int j = 0; j < kPer; ++j)
                if (tid + j * kSelThreads < n_above) mark(av[j], seg);
        }
        if (cached) {
#pragma unroll 1
            for (uint32_t c = tid; c < n_cand; c += kSelThreads) {
                const unsigned long long v = s_cand[c];
                if ((v & fmask) >= prefix) mark(~static_cast<uint32_t>(v), seg);
            }
        } else {
            constexpr int kB = 8;                       // candidate loads in flight per thread
#pragma unroll 1
            for (uint32_t c0 = tid; c0 < n_cand; c0 += kSelThreads * kB) {
                unsigned long long cv[kB];
#pragma unroll
                for (int j = 0; j < kB; ++j) {
                    const uint32_t c = c0 + j * kSelThreads;
                    cv[j] = c < n_cand ? __ldcg(w.cand + c) : 0ull;
                }
#pragma unroll
                for (int j = 0; j < kB; ++j)
                    if (c0 + j * kSelThreads < n_cand && (cv[j] & fmask) >= prefix)
                        mark(~static_cast<uint32_t>(cv[j]), seg);
            }
        }
        __syncthreads();
        const bool rotated = wpt == static_cast<uint32_t>(kWpt);
        const uint4* s_b4 = reinterpret_cast<const uint4*>(s_bits);
        // this thread's words: count and nonzero mask (bit q: word q)
        uint32_t cnt = 0, nz = 0;
        if (rotated) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v4 = s_b4[slot_of(tid, j)];
                cnt += __popc(v4.x) + __popc(v4.y) + __popc(v4.z) + __popc(v4.w);
                nz |= ((v4.x ? 1u : 0u) | (v4.y ? 2u : 0u) | (v4.z ? 4u : 0u) | (v4.w ? 8u : 0u)) << (4 * j);
            }
        } else {
            for (uint32_t q = 0; q < wpt; ++q) {
                const uint32_t x = s_bits[tid * wpt + q];
                cnt += __popc(x);
                nz |= (x ? 1u : 0u) << q;
            }
        }
        const uint32_t incl = block_incl_scan(cnt, sh_warp);
        if (tid == kSelThreads - 1) s_tot = incl;
        uint32_t pos = written + incl - cnt;
        {
            // one loop iteration per set bit of this thread (not per word and bit, which
            // would make a warp run the sum over words of its lanes' maxima)
            uint32_t bits = 0u, eb = 0u;
#pragma unroll 1
            for (;;) {
                if (bits == 0u) {
                    if (nz == 0u) break;
                    const uint32_t q = static_cast<uint32_t>(__ffs(nz) - 1);
                    nz &= nz - 1u;
                    bits = rotated ? s_bits[4 * slot_of(tid, q >> 2) + (q & 3u)] : s_bits[tid * wpt + q];
                    eb = static_cast<uint32_t>((seg + static_cast<size_t>(tid) * wpt + q) * 32);
                }
                const uint32_t e = eb + static_cast<uint32_t>(__ffs(bits) - 1);
                bits &= bits - 1u;
                if (pos < kk) orow[pos] = static_cast<int32_t>(e);
                ++pos;
            }
        }
        __syncthreads();
        written += s_tot;
        __syncthreads();
    }
    const uint32_t cnt_out = min(written, kk);
    for (uint32_t j = cnt_out + tid; j < static_cast<uint32_t>(k); j += kSelThreads) orow[j] = -1;
    if (tid == 0) count[r] = static_cast<int32_t>(cnt_out);
}

}  // namespace wide

}  // namespace

// few long rows, or rows too long for a 16-block cluster
bool topk_wide_preferred(int R, int64_t Nc_cap) {
    if (R <= 0 || Nc_cap < 8192) return false;
    return Nc_cap > 16 * kSliceMax || static_cast<int64_t>(R) * ceil_div(Nc_cap, kSlicePref) <= sm_count();
}

size_t topk_wide_ws_bytes(int R, int64_t Nc_cap) {
    return static_cast<size_t>(R) * wide::layout(Nc_cap).row_bytes;
}

// clear each row's histogram and header
int topk_wide_clear(void* ws, int R, int64_t Nc_cap, cudaStream_t st) {
    const wide::Layout L = wide::layout(Nc_cap);
    cudaError_t e = cudaMemset2DAsync(ws, L.row_bytes, 0, L.clear_bytes, static_cast<size_t>(R), st);
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    return HCA_OK;
}

// row r's key histogram (u32[2048]) starts at ws + r * stride u32 words
uint32_t* topk_wide_hist(void* ws, int64_t Nc_cap, int64_t* stride_u32) {
    *stride_u32 = static_cast<int64_t>(wide::layout(Nc_cap).row_bytes / 4);
    return static_cast<uint32_t*>(ws);
}

// scores per CTA: about one CTA per SM over all rows (hist_kernel), or at most
// one per two SMs (select_kernel: R * floor(SMs / 2 / R) CTAs, which fit in one
// wave beside a concurrent attention launch on the other SMs), whole steps
static int64_t wide_chunk(int R, int64_t Nc_cap, int per_step, int sms_per_cta = 1) {
    const int64_t ctas_per_row = sms_per_cta > 1 ? std::max<int64_t>(1, (sm_count() / sms_per_cta) / R)
                                                 : std::max<int64_t>(1, ceil_div(sm_count(), R));
    int64_t chunk = ceil_div(Nc_cap, ctas_per_row);
    chunk = std::max<int64_t>(per_step, ceil_div(chunk, per_step) * per_step);
    return std::min<int64_t>(chunk, static_cast<int64_t>(wide::kMaxIt) * per_step);
}

// CTAs left for a dense decode attention beside the decode select of B rows: the
// SMs that the select's B * floor(SMs / 2 / B) CTAs leave, at least half of them
int dense_beside_select(int B) {
    const int sm = sm_count();
    const int sel = B * std::max(1, (sm / 2) / std::max(B, 1));
    return std::max(sm / 2, sm - sel);
}

// select + resolve, given the rows' histograms (by hist_kernel or by the indexer);
// bf16: the scores are bf16 bit patterns (uint16)
int topk_wide_select(const void* scores, const int32_t* q_pos, int R, int64_t Nc_cap, int m, int k,
                     int32_t* idx, int32_t* count, void* ws, cudaStream_t st, bool bf16) {
    static bool attr_set[2][64] = {{false}, {false}};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[bf16][dev]) {
        const cudaError_t e =
            bf16 ? cudaFuncSetAttribute(wide::select_kernel<uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(wide::kSelSmem))
                 : cudaFuncSetAttribute(wide::select_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(wide::kSelSmem));
        if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
        attr_set[bf16][dev] = true;
    }
    const int64_t chunk = wide_chunk(R, Nc_cap, wide::kSelThreads, 2);
    const dim3 grid(static_cast<unsigned>(ceil_div(Nc_cap, chunk)), static_cast<unsigned>(R));
    // programmatic launch: the CTAs are placed while the histogram producer finishes
    const cudaError_t le =
        bf16 ? launch_pdl(wide::select_kernel<uint16_t>, grid, dim3(wide::kSelThreads), wide::kSelSmem, st,
                          static_cast<const uint16_t*>(scores), q_pos, Nc_cap, m, k, chunk, static_cast<uint8_t*>(ws),
                          idx, count)
             : launch_pdl(wide::select_kernel<float>, grid, dim3(wide::kSelThreads), wide::kSelSmem, st,
                          static_cast<const float*>(scores), q_pos, Nc_cap, m, k, chunk, static_cast<uint8_t*>(ws),
                          idx, count);
    if (le != cudaSuccess) { set_last_cuda_error(static_cast<int>(le)); return HCA_ERR_CUDA; }
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

int topk_wide_launch(const void* scores, const int32_t* q_pos, int R, int64_t Nc_cap, int m, int k,
                     int32_t* idx, int32_t* count, void* ws, cudaStream_t st, bool bf16) {
    const int rc = topk_wide_clear(ws, R, Nc_cap, st);
    if (rc != HCA_OK) return rc;
    const int64_t chunk = wide_chunk(R, Nc_cap, wide::kThreads * 8);
    const dim3 grid(static_cast<unsigned>(ceil_div(Nc_cap, chunk)), static_cast<unsigned>(R));
    if (bf16)
        wide::hist_kernel<uint16_t><<<grid, wide::kThreads, 0, st>>>(static_cast<const uint16_t*>(scores), q_pos,
                                                                    Nc_cap, m, chunk, static_cast<uint8_t*>(ws));
    else
        wide::hist_kernel<float><<<grid, wide::kThreads, 0, st>>>(static_cast<const float*>(scores), q_pos, Nc_cap,
                                                                 m, chunk, static_cast<uint8_t*>(ws));
    HCA_CHECK_LAUNCH();
    return topk_wide_select(scores, q_pos, R, Nc_cap, m, k, idx, count, ws, st, bf16);
}

int topk_launch(const float* scores, const int32_t* q_pos, int R, int64_t Nc_cap, int m, int k,
                int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, cudaStream_t st) {
    if (R == 0) return HCA_OK;
    if (topk_wide_preferred(R, Nc_cap) && ws != nullptr && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0 &&
        ws_bytes >= topk_wide_ws_bytes(R, Nc_cap) && R <= 65535 && Nc_cap <= 0x7FFFFFFFLL)
        return topk_wide_launch(scores, q_pos, R, Nc_cap, m, k, idx, count, ws, st, false);
    if (Nc_cap > 16 * kSliceMax) return HCA_ERR_WORKSPACE;   // only the workspace path takes such rows
    if (g_max_cluster == 0) {
        // probe once whether 16-CTA clusters of this kernel fit the device
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSliceMax * sizeof(uint32_t)));
        if (e == cudaSuccess) e = cudaFuncSetAttribute(topk_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        cudaLaunchConfig_t pc = {};
        pc.gridDim = dim3(16);
        pc.blockDim = dim3(kThreads);
        pc.dynamicSmemBytes = static_cast<size_t>(kSlicePref) * sizeof(uint32_t);
        cudaLaunchAttribute pa[1];
        pa[0].id = cudaLaunchAttributeClusterDimension;
        pa[0].val.clusterDim.x = 16; pa[0].val.clusterDim.y = 1; pa[0].val.clusterDim.z = 1;
        pc.attrs = pa; pc.numAttrs = 1;
        int n_clusters = 0;
        if (e != cudaSuccess || cudaOccupancyMaxActiveClusters(&n_clusters, topk_kernel<16>, &pc) != cudaSuccess)
            n_clusters = 0;
        cudaGetLastError();
        g_max_cluster = n_clusters > 0 ? 16 : 8;
    }
    // smallest cluster whose slices fit; for few rows, spread a row over more CTAs
    int CL = 1;
    while (ceil_div(Nc_cap, CL) > kSliceMax) CL *= 2;
    const int64_t want = ceil_div(2LL * sm_count(), R);
    while (CL < g_max_cluster && CL < want && ceil_div(Nc_cap, CL * 2) >= 1024 &&
           ceil_div(Nc_cap, CL) > kSlicePref / 4) CL *= 2;
    if (CL > g_max_cluster) return HCA_ERR_UNSUPPORTED;
    const int64_t slice = Nc_cap == 0 ? 1 : ceil_div(Nc_cap, CL);
    cudaError_t e;
    switch (CL) {
        case 1: e = launch_cl<1>(R, slice, scores, q_pos, Nc_cap, m, k, idx, count, st); break;
        case 2: e = launch_cl<2>(R, slice, scores, q_pos, Nc_cap, m, k, idx, count, st); break;
        case 4: e = launch_cl<4>(R, slice, scores, q_pos, Nc_cap, m, k, idx, count, st); break;
        case 8: e = launch_cl<8>(R, slice, scores, q_pos, Nc_cap, m, k, idx, count, st); break;
        default: e = launch_cl<16>(R, slice, scores, q_pos, Nc_cap, m, k, idx, count, st); break;
    }
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

}  // namespace hca
