// topk.cu -- exact top-k of index scores per query.
//
// "DeepSeek V4: Towards Highly Efficient Million Token Context Intelligence"
// (papers.chlience.com reading note), section 7: the selected set is the
// entries whose index score is in Top-k(I_{t,:}).  Ties go to the lower
// entry index; the output lists the chosen indices in ascending order.
//
// One row (one query's scores) is split over a thread-block cluster of CL
// CTAs (CL = 1..16), each holding a slice of at most 32768 scores in shared
// memory as order-preserving 32-bit keys.  A 3-digit (11/11/10-bit) radix
// select finds the exact key T of the k-th largest score: every CTA builds
// a digit histogram of the keys that still match the prefix, the cluster
// barrier publishes them, and every CTA sums all CL histograms through
// distributed shared memory and takes the same decision.  The selection is
// then: every key > T, plus the first `need` keys == T in index order.  A
// warp-ballot ordered compaction writes the indices in ascending order, with
// per-warp and per-CTA offsets from block and cluster prefix sums.
// Hardware cluster barriers order everything: no flag spinning.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace hca {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int64_t kSliceMax = 32768;

// Larger key = larger score; +0 and -0 map to the same key.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kThreads)
topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ q_pos, int64_t Nc_cap,
            int m, int k, int64_t slice, int32_t* __restrict__ idx, int32_t* __restrict__ count) {
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int64_t row = blockIdx.x / CL;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    extern __shared__ uint32_t keys[];                 // [slice]
    __shared__ uint32_t hist[2][kBins];
    __shared__ int pub[2];                             // published: ties, selected
    __shared__ int w_ties[kWarps], w_above[kWarps], w_sel[kWarps];
    __shared__ int bc[4];

    int64_t E = (static_cast<int64_t>(q_pos[row]) + 1) / m;
    E = E < 0 ? 0 : (E > Nc_cap ? Nc_cap : E);
    const int K = static_cast<int>(E < k ? E : k);
    const bool take_all = (K == E);
    const int64_t lo = static_cast<int64_t>(rank) * slice;
    const int64_t hi_ = lo + slice < E ? lo + slice : E;
    const int n = hi_ > lo ? static_cast<int>(hi_ - lo) : 0;

    const float* src = scores + row * Nc_cap + lo;
    for (int i = tid; i < n; i += kThreads) keys[i] = order_key(src[i]);
    __syncthreads();

    uint32_t T = 0;
    int need = 0;
    if (!take_all) {
        uint32_t prefix = 0, pmask = 0;
        need = K;
#pragma unroll 1
        for (int dgt = 0; dgt < 3; ++dgt) {
            const int sh = dgt == 0 ? 21 : (dgt == 1 ? 10 : 0);
            const uint32_t dm = dgt == 2 ? 0x3FFu : 0x7FFu;
            uint32_t* h = hist[dgt & 1];
            for (int i = tid; i < kBins; i += kThreads) h[i] = 0;
            __syncthreads();
            for (int i = tid; i < n; i += kThreads) {
                const uint32_t kk = keys[i];
                if ((kk & pmask) == prefix) atomicAdd(&h[(kk >> sh) & dm], 1u);
            }
            cluster.sync();
            // thread t owns bins 4t .. 4t+3 of the cluster-wide histogram
            uint32_t c4[4] = {0, 0, 0, 0};
            for (int r = 0; r < CL; ++r) {
                const uint32_t* rh = cluster.map_shared_rank(h, r);
#pragma unroll
                for (int j = 0; j < 4; ++j) c4[j] += rh[tid * 4 + j];
            }
            // exclusive suffix sum (bins above mine) across threads, high bins first
            const int mine = static_cast<int>(c4[0] + c4[1] + c4[2] + c4[3]);
            const int rw = kWarps - 1 - warp, rl = 31 - lane;     // reversed order
            int v = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_down_sync(0xffffffffu, v, o);  // lanes above (higher bins)
                if (rl >= o) v += u;
            }
            // v = inclusive sum over lanes >= lane in this warp
            if (lane == 0) w_sel[warp] = v;
            __syncthreads();
            int above_w = 0;
            for (int w2 = warp + 1; w2 < kWarps; ++w2) above_w += w_sel[w2];
            (void)rw;
            const int above = above_w + v - mine;                   // count in bins above my 4
            // find the bin holding the need-th largest
            int acc = above;
#pragma unroll
            for (int j = 3; j >= 0; --j) {
                const int cj = static_cast<int>(c4[j]);
                if (acc < need && acc + cj >= need) { bc[0] = tid * 4 + j; bc[1] = acc; }
                acc += cj;
            }
            __syncthreads();
            prefix |= static_cast<uint32_t>(bc[0]) << sh;
            pmask |= dm << sh;
            need -= bc[1];
            __syncthreads();
        }
        T = prefix;
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
    if (lane == 0) { w_ties[warp] = ties; w_above[warp] = above; }
    __syncthreads();
    if (tid == 0) {
        int t = 0;
        for (int w2 = 0; w2 < kWarps; ++w2) t += w_ties[w2];
        pub[0] = t;
    }
    cluster.sync();
    int tie_base = 0;                                  // ties in lower CTAs and lower warps
    for (int r = 0; r < rank; ++r) tie_base += *cluster.map_shared_rank(&pub[0], r);
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
    int out_pos = 0;
    for (int r = 0; r < rank; ++r) out_pos += *cluster.map_shared_rank(&pub[1], r);
    for (int w2 = 0; w2 < warp; ++w2) out_pos += w_sel[w2];

    int32_t* orow = idx + row * k;
    int tie_rank = tie_base;
    const uint32_t lt = (1u << lane) - 1u;
    for (int j = ws; j < we; j += 32) {
        const int i = j + lane;
        const uint32_t kk = i < we ? keys[i] : 0u;
        const bool in = i < we;
        const bool is_tie = in && !take_all && kk == T;
        const uint32_t tb = __ballot_sync(0xffffffffu, is_tie);
        const bool take = in && (take_all || kk > T || (is_tie && tie_rank + __popc(tb & lt) < need));
        const uint32_t sb = __ballot_sync(0xffffffffu, take);
        if (take) orow[out_pos + __popc(sb & lt)] = static_cast<int32_t>(lo + i);
        out_pos += __popc(sb);
        tie_rank += __popc(tb);
    }
    if (rank == 0) {
        for (int j = K + tid; j < k; j += kThreads) orow[j] = -1;
        if (tid == 0) count[row] = K;
    }
    cluster.sync();   // no CTA leaves while a peer may still read its shared memory
}

}  // namespace

int topk_launch(const float* scores, const int32_t* q_pos, int R, int64_t Nc_cap, int m, int k,
                int32_t* idx, int32_t* count, cudaStream_t st) {
    if (R == 0) return HCA_OK;
    int CL = 1;
    while (ceil_div(Nc_cap, CL) > kSliceMax) CL *= 2;
    if (CL > 16) return HCA_ERR_UNSUPPORTED;
    const int64_t slice = Nc_cap == 0 ? 1 : ceil_div(Nc_cap, CL);
    const size_t smem = static_cast<size_t>(slice) * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSliceMax * sizeof(uint32_t)));
    if (e == cudaSuccess && CL > 8)
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(static_cast<int64_t>(R) * CL));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, topk_kernel, scores, q_pos, Nc_cap, m, k, slice, idx, count);
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

}  // namespace hca
