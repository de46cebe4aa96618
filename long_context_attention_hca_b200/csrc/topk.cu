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

}  // namespace

int topk_launch(const float* scores, const int32_t* q_pos, int R, int64_t Nc_cap, int m, int k,
                int32_t* idx, int32_t* count, cudaStream_t st) {
    if (R == 0) return HCA_OK;
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
