// attention_tc.cu -- core attention of CSA and HCA on the sm_100a tensor
// cores (tcgen05 + TMEM), for decode (split-K) and chunked prefill, d = 512,
// H = 64 query heads sharing one KV head.
//
// "DeepSeek V4: Towards Highly Efficient Million Token Context Intelligence"
// (papers.chlience.com reading note), section 7: shared key-value MQA (the
// compressed entry is both key and value) plus the sliding-window branch;
// section 8: HCA attends densely to every compressed entry; section 9: FP8
// entries with BF16 RoPE dims.  One joint softmax over compressed and window
// keys.
//
// One CTA = one (query token, split): 64 heads against a run of 64-key tiles.
//   S    = Q . K^T      M = 64 heads (TMEM lanes 32w + r, r < 16), N = 64 keys,
//                       K = 512; Q (fp16, K-major SW128) stays in shared memory.
//   O^T += V^T . P^T    M = 128 output dims (4 M-tiles), N = 64 heads,
//                       K = 64 keys; V^T is the key tile itself read MN-major,
//                       P^T the softmax probabilities stored K-major.
// TMEM: S in NBUF buffers, each two 64-column partial sums (K halves), + O^T
// (4 x 64 columns): all 512 columns.
// Warp roles (768 threads):
//   warps 0-3   softmax: head h = 16 w + (lane & 15); lanes 0-15 take keys
//               0..31 of the tile, lanes 16-31 keys 32..63; online softmax
//               in base 2 with a lazy rescale (O^T and l are rescaled only
//               when a head's running max grows by more than 8, so P <= 2^8
//               in fp16).  They store P^T and hand it to the PV issuers
//               through an mbarrier (no barrier among themselves after the
//               stores, so the rescale state is double-buffered by tile
//               parity: a warp may run one tile ahead).
//   warps 4-19  producers: tile i goes to key buffer i % 2 (FP8 code x
//               scale -> fp16, bf16 -> fp16).  Warp w converts column block
//               w % 8 (64 dims) of key rows 32 (w / 8) .. + 31: lane l takes
//               16-dim unit l / 8 of that block and rows l % 8 + 8 j, so the
//               eight lanes that write one 16-byte chunk position hit eight
//               different swizzled bank groups.  Each thread issues the raw
//               loads of tile i + 1 as soon as tile i is stored (before it
//               waits for the buffer), and prefetches the gather indices one
//               tile ahead.
//   warps 20-21 QK issue: lane 0 of warp 20 + c issues half c of every
//               tile's QK (dims 256 c .. + 255, 16 MMAs) into its own
//               accumulator; the softmax adds the two.  One thread issues a
//               tcgen05.mma about every 70 clocks whatever its shape, so the
//               issue is spread over warps on different sub-partitions.
//   warps 22-23 PV issue: lane 0 of warp 22 + c issues M-tiles 2c, 2c + 1 of
//               O^T += V^T . P^T once the softmax warps have stored P(i),
//               then commits the P and key buffers' release (tcgen05.commit
//               tracks the issuing thread's own MMAs: the release barriers
//               count two arrivals).
//   All threads load Q (bf16 -> fp16) at the start, every load in flight at once.
//   Output: warps 0-15 (four per TMEM lane quarter, one M-tile each, one
//   output dim per thread).  One split: O / l as bf16, the RoPE dims rotated
//   back (about 5x shorter than the softmax warps alone: 32K clocks of a
//   prefill CTA's 120K were that epilogue).  Several splits: O / l as fp16
//   with heads in fours ([HP/4][D][4]), so a warp's 32 lanes (consecutive
//   dims) write 256 contiguous bytes per store.
// Per 64-key tile the MMAs read 128 KB of shared memory (Q and K for QK) and
// 96 KB (V^T and P, four M-tiles, for PV) and the stores write 72 KB: at
// 128 B per clock that is ~2300 clocks, the bound of this data flow.
// Launches are programmatic (the kernel waits for its stream predecessor
// before its first read, except for the query of a sparse launch made with the
// early-query knob on, which its caller guarantees complete before that
// predecessor started) and trigger the combine once their outputs are stored.
// Every mbarrier wait is bounded; a timeout sets the device error word,
// raises the CTA's abort flag, drains the issued MMAs and frees TMEM.
#include <mutex>

#include "common.cuh"

namespace hca {

__device__ int g_tc_device_error = 0;

namespace tc {

constexpr int D = 512;
constexpr int HP = 64;
constexpr int TK = 64;                       // keys per tile
constexpr int NBUF = 2;                      // key tiles (and S tiles) in flight
constexpr int NSOFT = 4, NPROD = 16, NISSUE = 2, NPV = 2;
constexpr int NWARPS = NSOFT + NPROD + NISSUE + NPV;
constexpr int NTHREADS = NWARPS * 32;        // 768
constexpr int ROWS_PER_THREAD = TK / NPROD;  // key rows a producer thread converts (4)
constexpr int QBLK = 8192;                   // Q column block: 64 head rows x 128 B (SW128)
constexpr int KBLK = TK * 128;               // key column block: 64 key rows x 128 B
constexpr int PBLK = 64 * 128;               // P^T: 64 head rows x 64 keys fp16 (one SW128 block)
constexpr int Q_OFF = 0;                     // 8 column blocks (64 KB)
constexpr int K_OFF = 8 * QBLK;              // NBUF buffers x 8 column blocks (2 x 64 KB)
constexpr int P_OFF = K_OFF + NBUF * 8 * KBLK;   // 2 P^T buffers
constexpr int SMEM_BYTES = P_OFF + 2 * PBLK + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t S_COL = 0;                // S buffer b, half c (of K = 512) at columns 64 (2 b + c)
constexpr uint32_t O_COL = NBUF * 2 * TK;    // O^T M-tile mt at 256 + 64 mt
constexpr float RESCALE_THRESHOLD = 8.0f;    // log2 units
constexpr long long WAIT_LIMIT = 1ll << 24;  // polls before a wait is declared stuck

struct Params {
    const uint16_t* q;          // [units][H][D] bf16
    int H;
    const uint8_t* codes;
    const float* scales;
    const uint16_t* rope;
    int64_t cap;
    int prefill;
    const int32_t* idx;
    int idx_stride;
    const int32_t* n_comp;
    int dense_m;
    int p0;
    const uint16_t* win;
    int W;
    float scale_log2;
    int n_splits, tiles_per_split;
    uint16_t* out;
    float* lse;
    uint16_t* part_o;           // [units][splits][HP/4][D][4] fp16: the split's O / l, heads in fours
    float* part_ml;             // [units][splits][2][HP]: running max (base 2), l
    // section 9 extras (each null when off)
    const float* q_norm_w;      // [D] query-head RMSNorm weight
    float norm_eps;
    const float* sink;          // [HP] sink logit per head (natural log)
    const float* inv_freq;      // [32] RoPE frequencies of the 64 RoPE dims
    const int32_t* q_pos;       // decode: [units] query positions
    const int32_t* win_len;     // decode: [units] valid window rows (<= W), or null: W
    int q_early;                // the query may be read before the wait on the previous kernel
};

constexpr int D_ROPE = 64;
constexpr float LOG2E = 1.4426950408889634f;

// Position of a unit's query token: its sequence's query (decode), p0 + unit (prefill).
__device__ __forceinline__ int64_t unit_pos(const Params& p, int64_t u) {
    return p.prefill ? static_cast<int64_t>(p.p0) + u : (p.q_pos ? static_cast<int64_t>(p.q_pos[u]) : 0);
}

// cos / sin of RoPE pair i at position t (fp64 angle t * f_i, exact; fp32 out)
__device__ __forceinline__ void rope_cs(const float* inv_freq, int i, int64_t t, float& c, float& s) {
    double sn, cs;
    sincos(static_cast<double>(t) * static_cast<double>(__ldg(inv_freq + i)), &sn, &cs);
    c = static_cast<float>(cs);
    s = static_cast<float>(sn);
}

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(dst), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(n) : "memory"); }

#define TMEM_LD16(taddr, r, o)                                                                                     \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];" \
                 : "=r"(r[o + 0]), "=r"(r[o + 1]), "=r"(r[o + 2]), "=r"(r[o + 3]), "=r"(r[o + 4]), "=r"(r[o + 5]),    \
                   "=r"(r[o + 6]), "=r"(r[o + 7]), "=r"(r[o + 8]), "=r"(r[o + 9]), "=r"(r[o + 10]), "=r"(r[o + 11]),  \
                   "=r"(r[o + 12]), "=r"(r[o + 13]), "=r"(r[o + 14]), "=r"(r[o + 15])                                \
                 : "r"(taddr))
#define TMEM_ST16(taddr, r, o)                                                                                     \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" \
                 :: "r"(taddr), "r"(r[o + 0]), "r"(r[o + 1]), "r"(r[o + 2]), "r"(r[o + 3]), "r"(r[o + 4]),            \
                   "r"(r[o + 5]), "r"(r[o + 6]), "r"(r[o + 7]), "r"(r[o + 8]), "r"(r[o + 9]), "r"(r[o + 10]),         \
                   "r"(r[o + 11]), "r"(r[o + 12]), "r"(r[o + 13]), "r"(r[o + 14]), "r"(r[o + 15]) : "memory")
#define TMEM_LD32(taddr, r)                                                                                        \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"    \
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                           \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),      \
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), \
                   "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),          \
                   "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),          \
                   "=r"(r[30]), "=r"(r[31])                                                                         \
                 : "r"(taddr))
// 16 TMEM lanes x 32 columns, twice: threads 0-15 read lanes base + t at columns
// c .. c + 31, threads 16-31 the same lanes at columns c + 32 .. c + 63 (the M = 64
// accumulator layout keeps a warp's 16 rows in the first 16 lanes of its quarter)
#define TMEM_LD_16X32BX2_32(taddr, r)                                                                              \
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15," \
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"                       \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),      \
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), \
                   "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),          \
                   "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),          \
                   "=r"(r[30]), "=r"(r[31])                                                                         \
                 : "r"(taddr))
// the same with 16 columns per half: threads 0-15 columns c .. c + 15, threads
// 16-31 columns c + 32 .. c + 47
#define TMEM_LD_16X32BX2_16(taddr, r)                                                                              \
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 32;" \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),      \
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]) \
                 : "r"(taddr))
// 2^x with the special-function unit (approximate; x = -inf gives +0)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// shared-memory matrix descriptor, 128-byte swizzle (sm_100 format)
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// instruction descriptor, kind::f16: fp16 A and B, fp32 accumulator
__device__ __forceinline__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
// byte offset of (row, 16-byte chunk c in 0..7) inside an SW128 column block
__device__ __forceinline__ uint32_t sw128(int row, int c) {
    return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((c ^ (row & 7)) << 4));
}

struct UnitKeys {
    int n_c, n_w;
    const int32_t* ent;
    int64_t kv_row0;
    const uint16_t* wrow;
};

__device__ __forceinline__ UnitKeys unit_keys(const Params& p, int64_t u) {
    UnitKeys k;
    if (!p.prefill) {
        const int nc = p.n_comp[u];
        k.n_c = nc < 0 ? 0 : nc;
        k.ent = p.idx ? p.idx + u * p.idx_stride : nullptr;
        k.kv_row0 = u * p.cap;
        k.wrow = p.win + static_cast<size_t>(u) * p.W * D;
        k.n_w = p.W;
        if (p.win_len) {
            const int wl = p.win_len[u];
            k.n_w = wl < 0 ? 0 : (wl > p.W ? p.W : wl);
        }
    } else {
        const int64_t pos = p.p0 + u;
        if (p.idx) {
            const int nc = p.n_comp[u];
            k.n_c = nc < 0 ? 0 : nc;
            k.ent = p.idx + u * p.idx_stride;
        } else {
            const int64_t e = (pos + 1) / p.dense_m;
            k.n_c = static_cast<int>(e > p.cap ? p.cap : e);
            k.ent = nullptr;
        }
        k.kv_row0 = 0;
        const int64_t first = pos - (p.W - 1) > 0 ? pos - (p.W - 1) : 0;
        k.wrow = p.win + static_cast<size_t>(first - (p.p0 - (p.W - 1))) * D;
        k.n_w = static_cast<int>(pos - first + 1);
    }
    return k;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
    return pack_half2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

// Bounded wait; returns false on timeout (and records it).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    for (long long it = 0; it < WAIT_LIMIT; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 1023) == 1023 && *abort_flag) return false;
    }
    *abort_flag = 1;
    atomicExch(&g_tc_device_error, 1);
    return false;
}

// EX: the section 9 extras are compiled in (query RMSNorm / RoPE, sink, output
// RoPE); without them the kernel carries none of that code.
template <bool EX>
__global__ void __launch_bounds__(NTHREADS, 1) attn_tc_kernel(Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar_kempty[NBUF], bar_kfull[NBUF], bar_sfull[NBUF], bar_pready[2], bar_pempty[2],
        bar_drain;
    __shared__ uint32_t tmem_base_slot;
    // rescale factors and flags, double-buffered by tile parity: with no barrier
    // after the P stores a warp may run one tile ahead of the others
    __shared__ float s_alpha[2][HP], s_rl[HP];
    __shared__ int s_resc_w[2][NSOFT];
    __shared__ volatile int s_abort;
    __shared__ float s_qr[HP];                       // 1 / rms of each query head (query RMSNorm)
    __shared__ float s_cos[D_ROPE / 2], s_sin[D_ROPE / 2];   // RoPE of the unit's position

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t u = blockIdx.x;
    const int split = blockIdx.y;
    // the query, converted (and, with the extras, normalised and rotated) into its
    // shared-memory operand; before the wait on the previous kernel when the launch
    // says that the query was complete before that kernel started (p.q_early)
    auto load_q = [&]() {
        // Q -> fp16, K-major SW128: column block cb = dims 64cb.., row = head; all of
        // a thread's loads are issued before the first conversion
        constexpr int QV = HP * (D / 8);                      // 16-byte vectors of Q
        constexpr int QPT = (QV + NTHREADS - 1) / NTHREADS;   // per thread
        uint4 qv[QPT];
#pragma unroll
        for (int k = 0; k < QPT; ++k) {
            const int w = tid + k * NTHREADS, r = w / (D / 8), c = w % (D / 8);
            qv[k] = (w < QV && r < p.H)
                        ? __ldg(reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(u) * p.H + r) * D + c * 8))
                        : make_uint4(0, 0, 0, 0);
        }
        if (!EX || (p.q_norm_w == nullptr && p.inv_freq == nullptr)) {
#pragma unroll
            for (int k = 0; k < QPT; ++k) {
                const int w = tid + k * NTHREADS, r = w / (D / 8), c = w % (D / 8);
                if (w < QV)
                    *reinterpret_cast<uint4*>(smem + Q_OFF + (c >> 3) * QBLK + sw128(r, c & 7)) =
                        make_uint4(bf16x2_to_f16x2(qv[k].x), bf16x2_to_f16x2(qv[k].y), bf16x2_to_f16x2(qv[k].z),
                                   bf16x2_to_f16x2(qv[k].w));
            }
        } else {
            // section 9 extras of the query, in fp32 before the fp16 store: each head
            // RMS-normalised (partial sums of squares per 16-byte vector in the P
            // buffers, free until the softmax), its RoPE dims rotated to the unit's
            // position
            const int64_t tpos = unit_pos(p, u);
            if (p.inv_freq && tid < D_ROPE / 2) rope_cs(p.inv_freq, tid, tpos, s_cos[tid], s_sin[tid]);
            if (p.q_norm_w) {
                float* s_qss = reinterpret_cast<float*>(smem + P_OFF);       // [HP][D / 8]
#pragma unroll
                for (int k = 0; k < QPT; ++k) {
                    const int w = tid + k * NTHREADS;
                    if (w < QV) {
                        const uint32_t v4[4] = {qv[k].x, qv[k].y, qv[k].z, qv[k].w};
                        float ss = 0.0f;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float a = __uint_as_float(v4[i] << 16), b = __uint_as_float(v4[i] & 0xFFFF0000u);
                            ss += a * a + b * b;
                        }
                        s_qss[w] = ss;
                    }
                }
                __syncthreads();
                if (tid < HP) {
                    float ss = 0.0f;
                    for (int c = 0; c < D / 8; ++c) ss += s_qss[tid * (D / 8) + c];
                    s_qr[tid] = rsqrtf(ss / static_cast<float>(D) + p.norm_eps);
                }
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < QPT; ++k) {
                const int w = tid + k * NTHREADS, r = w / (D / 8), c = w % (D / 8);
                if (w < QV) {
                    const uint32_t v4[4] = {qv[k].x, qv[k].y, qv[k].z, qv[k].w};
                    float f[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        f[2 * i] = __uint_as_float(v4[i] << 16);
                        f[2 * i + 1] = __uint_as_float(v4[i] & 0xFFFF0000u);
                    }
                    if (p.q_norm_w) {
                        const float4 wa = __ldg(reinterpret_cast<const float4*>(p.q_norm_w + c * 8));
                        const float4 wb = __ldg(reinterpret_cast<const float4*>(p.q_norm_w + c * 8) + 1);
                        const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                        const float rr = s_qr[r];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = f[i] * rr * wv[i];
                    }
                    if (p.inv_freq && c * 8 >= D - D_ROPE) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int pi = (c * 8 - (D - D_ROPE)) / 2 + i;
                            const float a = f[2 * i], b = f[2 * i + 1], cs = s_cos[pi], sn = s_sin[pi];
                            f[2 * i] = a * cs - b * sn;
                            f[2 * i + 1] = a * sn + b * cs;
                        }
                    }
                    *reinterpret_cast<uint4*>(smem + Q_OFF + (c >> 3) * QBLK + sw128(r, c & 7)) =
                        make_uint4(pack_half2(f[0], f[1]), pack_half2(f[2], f[3]), pack_half2(f[4], f[5]),
                                   pack_half2(f[6], f[7]));
                }
            }
        }
    };
    if (p.q_early) load_q();
    pdl_wait();                                    // everything earlier in the stream is visible
    const UnitKeys uk = unit_keys(p, u);
    const int n_tot = uk.n_c + uk.n_w;
    const int n_tiles_all = (n_tot + TK - 1) / TK;
    const int t_begin = split * p.tiles_per_split;
    const int t_end = min(n_tiles_all, t_begin + p.tiles_per_split);
    const int n_tiles = t_end > t_begin ? t_end - t_begin : 0;
    const uint32_t sbase = smem_u32(smem);

    if (tid == 0) {
        for (int i = 0; i < NBUF; ++i) {
            mbar_init(smem_u32(&bar_kempty[i]), NPV);  // freed by the PV issuers
            mbar_init(smem_u32(&bar_kfull[i]), NPROD);  // one arrival per producer warp
            mbar_init(smem_u32(&bar_sfull[i]), NISSUE);   // both QK issuers
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bar_pready[i]), NSOFT);  // the softmax warps stored P
            mbar_init(smem_u32(&bar_pempty[i]), NPV);    // the PV issuers' MMAs completed
        }
        mbar_init(smem_u32(&bar_drain), NISSUE + NPV);   // the MMA-issuing threads
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) { tmem_alloc(smem_u32(&tmem_base_slot), TMEM_COLS); tmem_relinquish(); }
    // ---- producer state (warps 4-19), declared here so that the first tile's
    // gathers are in flight while every thread loads Q
    const bool producer = warp >= NSOFT && warp < NSOFT + NPROD;
    const int pw = warp - NSOFT;                   // 0..15
    const int c16 = (pw & 7) * 4 + (lane >> 3);    // this thread's 16-dim unit (same for all its keys)
    const int row0 = (pw >> 3) * 32 + (lane & 7);  // its rows: row0 + 8 j
    const int d0 = c16 * 16;
    const int dn = D - 64;
    int32_t ent_next[ROWS_PER_THREAD];
    auto fetch_ent = [&](int i, int32_t (&e)[ROWS_PER_THREAD]) {
#pragma unroll
        for (int j = 0; j < ROWS_PER_THREAD; ++j) {
            const int slot = (t_begin + i) * TK + row0 + 8 * j;
            e[j] = (i < n_tiles && slot < uk.n_c) ? (uk.ent ? uk.ent[slot] : slot) : -1;
        }
    };
    uint32_t raw[ROWS_PER_THREAD][8];
    float sc[ROWS_PER_THREAD];
    // raw loads of tile i (registers only: no buffer needed yet)
    auto load_tile = [&](int i, const int32_t (&ent)[ROWS_PER_THREAD]) {
        const int slot0 = (t_begin + i) * TK;
#pragma unroll
        for (int j = 0; j < ROWS_PER_THREAD; ++j) {
            const int r = row0 + 8 * j;
            const int slot = slot0 + r;
            sc[j] = 0.0f;
#pragma unroll
            for (int z = 0; z < 8; ++z) raw[j][z] = 0;
            if (i >= n_tiles) continue;
            if (slot < uk.n_c) {
                const int64_t e = ent[j];
                if (e >= 0 && e < p.cap) {
                    const int64_t er = uk.kv_row0 + e;
                    if (d0 < dn) {
                        const uint4 cv = __ldg(reinterpret_cast<const uint4*>(p.codes + er * dn + d0));
                        raw[j][0] = cv.x; raw[j][1] = cv.y; raw[j][2] = cv.z; raw[j][3] = cv.w;
                        sc[j] = __ldg(p.scales + er * (dn / 64) + d0 / 64);
                    } else {
                        const uint4* rp = reinterpret_cast<const uint4*>(p.rope + er * 64 + (d0 - dn));
                        const uint4 a = __ldg(rp), bq = __ldg(rp + 1);
                        raw[j][0] = a.x; raw[j][1] = a.y; raw[j][2] = a.z; raw[j][3] = a.w;
                        raw[j][4] = bq.x; raw[j][5] = bq.y; raw[j][6] = bq.z; raw[j][7] = bq.w;
                    }
                }
            } else if (slot < n_tot) {
                const uint4* rp = reinterpret_cast<const uint4*>(uk.wrow + static_cast<size_t>(slot - uk.n_c) * D + d0);
                const uint4 a = __ldg(rp), bq = __ldg(rp + 1);
                raw[j][0] = a.x; raw[j][1] = a.y; raw[j][2] = a.z; raw[j][3] = a.w;
                raw[j][4] = bq.x; raw[j][5] = bq.y; raw[j][6] = bq.z; raw[j][7] = bq.w;
            }
        }
    };
    if (producer) {
        int32_t ent0[ROWS_PER_THREAD];
        fetch_ent(0, ent0);
        load_tile(0, ent0);
        fetch_ent(1, ent_next);
    }
    if (!p.q_early) load_q();
    fence_async_smem();
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = tmem_base_slot;

    constexpr uint32_t id_qk = idesc_f16(64, TK, 0, 0);   // S[64 heads x 64 keys]
    constexpr uint32_t id_pv = idesc_f16(128, HP, 1, 0);
    if (warp >= NSOFT + NPROD + NISSUE) {
        // ------------------------------------------------------------ PV issue
        // O^T += V^T . P^T, V^T read MN-major from the key tile: dims in atoms of 64
        // (column blocks, KBLK apart), keys in atoms of 8 rows (1024 B apart).  Lane 0
        // of warp 22 + c issues M-tiles 2 c and 2 c + 1 (output dims 256 c .. + 255),
        // off the softmax warps' path.
        const int c = warp - (NSOFT + NPROD + NISSUE);
        if (lane == 0) {
            for (int i = 0; i < n_tiles; ++i) {
                const int b = i % NBUF, pb = i & 1;
                if (!wait_bar(smem_u32(&bar_pready[pb]), (i >> 1) & 1, &s_abort)) break;
                fence_after();
                const uint64_t vd = sdesc(sbase + K_OFF + b * 8 * KBLK, KBLK, 1024);
                const uint64_t pd = sdesc(sbase + P_OFF + pb * PBLK, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < TK / 16; ++kk)
#pragma unroll
                    for (int m2 = 0; m2 < 2; ++m2) {
                        const int mt = 2 * c + m2;
                        mma_f16(tmem + O_COL + mt * HP, vd + static_cast<uint32_t>((2 * mt * KBLK + kk * 2048) >> 4),
                                pd + static_cast<uint32_t>((kk * 32) >> 4), id_pv, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                mma_commit(smem_u32(&bar_pempty[pb]));
                mma_commit(smem_u32(&bar_kempty[b]));
            }
            mma_commit(smem_u32(&bar_drain));
        }
    } else if (warp >= NSOFT + NPROD) {
        // ------------------------------------------------------------ QK issue
        // Warp 20 + c issues half c of every tile's QK (dims 256 c .. 256 c + 255) into
        // its own accumulator: one thread issues an MMA every ~70 clocks whatever its
        // shape, so two issuers on two sub-partitions halve the QK time.
        const int c = warp - (NSOFT + NPROD);
        if (lane == 0) {
            const uint64_t qd = sdesc(sbase + Q_OFF, 16, 1024);
            for (int i = 0; i < n_tiles; ++i) {
                const int b = i % NBUF;
                if (!wait_bar(smem_u32(&bar_kfull[b]), (i / NBUF) & 1, &s_abort)) break;
                fence_after();
                const uint64_t kd = sdesc(sbase + K_OFF + b * 8 * KBLK, 16, 1024);
                const uint32_t dst = tmem + S_COL + (2 * b + c) * TK;
                // descriptors differ per k-step only in the start address (bits 0..13, units of 16 B)
#pragma unroll
                for (int k2 = 0; k2 < D / 32; ++k2) {
                    const int kk = c * (D / 32) + k2;
                    const uint32_t qo = static_cast<uint32_t>(((kk >> 2) * QBLK + (kk & 3) * 32) >> 4);
                    const uint32_t ko = static_cast<uint32_t>(((kk >> 2) * KBLK + (kk & 3) * 32) >> 4);
                    mma_f16(dst, qd + qo, kd + ko, id_qk, k2 > 0);
                }
                mma_commit(smem_u32(&bar_sfull[b]));
            }
            mma_commit(smem_u32(&bar_drain));
        }
    } else if (warp >= NSOFT) {
        // ------------------------------------------------------------ producers
        for (int i = 0; i < n_tiles; ++i) {
            const int b = i % NBUF, use = i / NBUF;
            const int slot0 = (t_begin + i) * TK;
            // key buffer b is free once PV(i - 2) has completed
            if (use >= 1 && !wait_bar(smem_u32(&bar_kempty[b]), (use - 1) & 1, &s_abort)) break;
            uint8_t* kb = smem + K_OFF + b * 8 * KBLK;
#pragma unroll
            for (int j = 0; j < ROWS_PER_THREAD; ++j) {
                const int r = row0 + 8 * j;
                const bool fp8 = slot0 + r < uk.n_c && d0 < dn;
                uint32_t h[8];
                if (fp8) {
                    const float s_ = sc[j];
                    if (s_ >= 6.103515625e-05f && s_ <= 65504.0f) {
                        // scale is a normal fp16: code (exact in fp16) x fp16(scale), one
                        // fp16 rounding per product, two elements per instruction
                        const uint32_t s2 = pack_half2(s_, s_);
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            h[2 * z] = hmul2_u32(e4m3x2_to_f16x2(static_cast<uint16_t>(raw[j][z] & 0xFFFFu)), s2);
                            h[2 * z + 1] = hmul2_u32(e4m3x2_to_f16x2(static_cast<uint16_t>(raw[j][z] >> 16)), s2);
                        }
                    } else {
                        // tiny, zero or huge scale: fp32 product, rounded once to fp16
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            const float2 a = unpack_half2(e4m3x2_to_f16x2(static_cast<uint16_t>(raw[j][z] & 0xFFFFu)));
                            const float2 bb = unpack_half2(e4m3x2_to_f16x2(static_cast<uint16_t>(raw[j][z] >> 16)));
                            h[2 * z] = pack_half2(a.x * s_, a.y * s_);
                            h[2 * z + 1] = pack_half2(bb.x * s_, bb.y * s_);
                        }
                    }
                } else {
#pragma unroll
                    for (int z = 0; z < 8; ++z) h[z] = bf16x2_to_f16x2(raw[j][z]);
                }
                // dims 16 c16 .. +15 = chunks 2 c16, 2 c16 + 1 of column block c16 / 4
                uint8_t* blk = kb + (c16 >> 2) * KBLK;
                const int c8 = (2 * c16) & 7;
                *reinterpret_cast<uint4*>(blk + sw128(r, c8)) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4*>(blk + sw128(r, c8 + 1)) = make_uint4(h[4], h[5], h[6], h[7]);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar_kfull[b]));
            // next tile's raw loads fly while this thread waits for its buffer
            int32_t ent[ROWS_PER_THREAD];
#pragma unroll
            for (int j = 0; j < ROWS_PER_THREAD; ++j) ent[j] = ent_next[j];
            load_tile(i + 1, ent);
            fetch_ent(i + 2, ent_next);
        }
    } else {
        // ------------------------------------------------------------ softmax (warps 0-3)
        // head h = 16 warp + (lane & 15); lanes 0-15 hold keys 0..31 of the tile, lanes
        // 16-31 keys 32..63 (S row h lives in TMEM lane 32 warp + (lane & 15)).
        const int h = warp * 16 + (lane & 15);
        const int kh = lane >> 4;
        float m_used = -INFINITY, l_run = 0.0f;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        bool ok = true;
        for (int i = 0; i < n_tiles; ++i) {
            const int b = i % NBUF, pb = i & 1;
            if (!wait_bar(smem_u32(&bar_sfull[b]), (i / NBUF) & 1, &s_abort)) { ok = false; break; }
            fence_after();
            const int nvalid = min(TK, n_tot - (t_begin + i) * TK);
            float v[32];
            float tmax = -INFINITY;
            {
                // row h, keys 32 kh .. 32 kh + 31: the sum of the two K-half accumulators
                uint32_t sr[32], s2[16];
                const uint32_t sa = lane_base + S_COL + (2 * b) * TK;
                TMEM_LD_16X32BX2_32(sa, sr);
                TMEM_LD_16X32BX2_16(sa + TK, s2);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(sr[j]) + __uint_as_float(s2[j]);
                TMEM_LD_16X32BX2_16(sa + TK + 16, s2);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) v[16 + j] = __uint_as_float(sr[16 + j]) + __uint_as_float(s2[j]);
                if (nvalid < TK) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (kh * 32 + j >= nvalid) v[j] = -INFINITY;
                }
                // maximum as a tree (depth 5 instead of a 32-long chain)
                float mx[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) mx[j] = fmaxf(v[j], v[j + 16]);
#pragma unroll
                for (int w2 = 8; w2 >= 1; w2 >>= 1)
#pragma unroll
                    for (int j = 0; j < w2; ++j) mx[j] = fmaxf(mx[j], mx[j + w2]);
                // the scale is positive (checked on the host): the maximum of the raw logits
                // times the scale is the maximum of the scaled ones
                tmax = mx[0] * p.scale_log2;
            }
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
            bool resc = false;
            float alpha = 1.0f;
            const float m_new = fmaxf(m_used, tmax);
            if (i == 0) {
                m_used = m_new;
            } else if (m_new > m_used + RESCALE_THRESHOLD) {
                resc = true;
                alpha = ex2(m_used - m_new);
                m_used = m_new;
                l_run *= alpha;
            }
            // probabilities in registers before any wait (fp16, the sum of the rounded values)
            uint32_t pk[16];
            float ps[16];
#pragma unroll
            for (int z = 0; z < 16; ++z) {
                pk[z] = pack_half2(ex2(fmaf(v[2 * z], p.scale_log2, -m_used)), ex2(fmaf(v[2 * z + 1], p.scale_log2, -m_used)));
                const float2 f = unpack_half2(pk[z]);
                ps[z] = f.x + f.y;
            }
            // row sum of the rounded probabilities as a tree
#pragma unroll
            for (int w2 = 8; w2 >= 1; w2 >>= 1)
#pragma unroll
                for (int j = 0; j < w2; ++j) ps[j] += ps[j + w2];
            float rs = ps[0];
            rs += __shfl_xor_sync(0xffffffffu, rs, 16);
            l_run += rs;
            if (lane < 16) s_alpha[i & 1][h] = alpha;
            const unsigned wr = __ballot_sync(0xffffffffu, resc);
            if (lane == 0) s_resc_w[i & 1][warp] = wr != 0u;
            // P buffer pb is free once PV(i-2) has completed
            if (i >= 2) {
                if (!wait_bar(smem_u32(&bar_pempty[pb]), ((i - 2) >> 1) & 1, &s_abort)) { ok = false; break; }
            }
            named_bar(1, NSOFT * 32);
            if (s_resc_w[i & 1][0] | s_resc_w[i & 1][1] | s_resc_w[i & 1][2] | s_resc_w[i & 1][3]) {
                // O^T must be stable: PV(i-1) complete
                if (i >= 1 && !wait_bar(smem_u32(&bar_pempty[(i - 1) & 1]), ((i - 1) >> 1) & 1, &s_abort)) { ok = false; break; }
                fence_after();
                // this thread owns TMEM lane 32 warp + lane = one output dim of each M-tile;
                // 16 head columns at a time (their factors stay in registers for the 4 M-tiles)
#pragma unroll 1
                for (int c0 = 0; c0 < HP; c0 += 16) {
                    float al[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) al[j] = s_alpha[i & 1][c0 + j];
#pragma unroll 1
                    for (int mt = 0; mt < 4; ++mt) {
                        uint32_t o[16];
                        TMEM_LD16(lane_base + O_COL + mt * HP + c0, o, 0);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * al[j]);
                        TMEM_ST16(lane_base + O_COL + mt * HP + c0, o, 0);
                    }
                }
                tmem_wait_st();
            }
            // P^T row h: keys 32 kh .. 32 kh + 31 are 16-byte chunks 4 kh .. 4 kh + 3
            uint8_t* pbuf = smem + P_OFF + pb * PBLK;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(pbuf + sw128(h, 4 * kh + c)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            // hand P(i) (and any rescale of O^T) to the PV issuers
            fence_async_smem();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar_pready[pb]));
        }
        // ---- epilogue: wait for the last PV, then 1 / l (and the split's (m, l)) for the output
        if (ok && n_tiles > 0) {
            ok = wait_bar(smem_u32(&bar_pempty[(n_tiles - 1) & 1]), ((n_tiles - 1) >> 1) & 1, &s_abort);
            fence_after();
        }
        const bool hrow = lane < 16;
        // the sink joins the denominator (relative to this split's running max)
        const float sink_l2 = (EX && p.sink) ? __ldg(p.sink + h) * LOG2E : -INFINITY;
        const float l_tot = (EX && p.sink && n_tiles > 0) ? l_run + ex2(sink_l2 - m_used) : l_run;
        const size_t uo = static_cast<size_t>(u);
        const float qnan = __int_as_float(0x7fc00000);
        if (p.n_splits == 1) {
            // the output itself (below, by warps 0-15): 1 / l of every head
            if (hrow) s_rl[h] = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
            if (p.lse && hrow && h < p.H) {
                const float none = (EX && p.sink) ? __ldg(p.sink + h) : -INFINITY;    // no keys: the sink alone
                p.lse[uo * p.H + h] = (l_run > 0.0f && ok) ? (m_used + log2f(l_tot)) * 0.69314718055994531f
                                                          : (ok ? none : qnan);
            }
        } else if (hrow) {
            const size_t ps = uo * p.n_splits + split;
            float* ml = p.part_ml + ps * 2 * HP;
            ml[h] = m_used;
            ml[HP + h] = ok ? l_run : qnan;
            s_rl[h] = l_run > 0.0f ? 1.0f / l_run : 0.0f;
        }
    }
    if (warp < 16) {
        // ---- output by warps 0-15: warp w reads TMEM lane quarter w % 4 (the lanes it
        // may access) of M-tile w / 4, i.e. one output dim per thread.  One split: that
        // dim of every head, O / l as bf16 (the RoPE dims rotated back), the 32 lanes
        // (consecutive dims) of a warp writing 64 contiguous bytes per head.  Several
        // splits: O / l as fp16, four heads (8 bytes) per store, 256 contiguous bytes a
        // warp.  The softmax warps have seen the last PV complete (their own wait, one
        // phase at a time); the barrier hands that on with 1 / l
        fence_before();
        named_bar(2, 16 * 32);                       // s_rl published, the last PV complete
        fence_after();
        const int qd = warp & 3, mt = warp >> 2;
        const int dim = mt * 128 + qd * 32 + lane;
        const uint32_t lb = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        const bool good = s_abort == 0;
        if (p.n_splits == 1) {
            const size_t uo = static_cast<size_t>(u);
            const bool rot = EX && p.inv_freq && dim >= D - D_ROPE;
            const int pi = rot ? (dim - (D - D_ROPE)) >> 1 : 0;
            const float cs = rot ? s_cos[pi] : 1.0f, sn = rot ? s_sin[pi] : 0.0f;
            const uint16_t qnan16 = 0x7FC0u;
#pragma unroll 1
            for (int c1 = 0; c1 < HP; c1 += 32) {
                uint32_t oa[32];
                if (n_tiles > 0) {
                    TMEM_LD16(lb + O_COL + mt * HP + c1, oa, 0);
                    TMEM_LD16(lb + O_COL + mt * HP + c1 + 16, oa, 16);
                    tmem_wait_ld();
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int hh = c1 + j;
                    float v = n_tiles > 0 ? __uint_as_float(oa[j]) * s_rl[hh] : 0.0f;
                    if (EX && p.inv_freq && mt == 3) {
                        // RoPE pair (dim, dim ^ 1) of neighbouring lanes
                        const float pv = __shfl_xor_sync(0xffffffffu, v, 1);
                        if (rot) v = (dim & 1) ? v * cs - pv * sn : v * cs + pv * sn;
                    }
                    if (hh < p.H)
                        p.out[(uo * p.H + hh) * D + dim] = good ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : qnan16;
                }
            }
        } else if (n_tiles > 0) {
            uint16_t* po = p.part_o + (static_cast<size_t>(u) * p.n_splits + split) * HP * D + static_cast<size_t>(dim) * 4;
#pragma unroll 1
            for (int c1 = 0; c1 < HP; c1 += 32) {
                uint32_t oa[32];
                TMEM_LD16(lb + O_COL + mt * HP + c1, oa, 0);
                TMEM_LD16(lb + O_COL + mt * HP + c1 + 16, oa, 16);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int hq = c1 + 4 * j;         // heads hq .. hq + 3
                    uint2 hv;
                    hv.x = good ? pack_half2(__uint_as_float(oa[4 * j]) * s_rl[hq], __uint_as_float(oa[4 * j + 1]) * s_rl[hq + 1])
                                : 0x7E007E00u;
                    hv.y = good ? pack_half2(__uint_as_float(oa[4 * j + 2]) * s_rl[hq + 2], __uint_as_float(oa[4 * j + 3]) * s_rl[hq + 3])
                                : 0x7E007E00u;
                    *reinterpret_cast<uint2*>(po + static_cast<size_t>(hq / 4) * D * 4) = hv;
                }
            }
        }
    }
    fence_before();
    __syncthreads();
    pdl_trigger();                                 // outputs stored: the combine may be scheduled
    if (warp == 0) {
        // every issued MMA has completed before TMEM is freed
        if (lane == 0)
            for (long long it = 0; it < WAIT_LIMIT; ++it)
                if (mbar_try_wait(smem_u32(&bar_drain), 0)) break;
        __syncwarp();
        fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Log-sum-exp combine of split partials (base-2 maxima): grid (unit, 16-dim
// block), 128 threads.  Per head: M = max of the live splits' maxima, split
// weight 2^(m_s - M) l_s (the partials are O_s / l_s), L = their sum (+ the
// sink); out = sum_s weight_s o_s / L.  Thread t sums heads 4 (t / 8) .. + 3
// at dims 16 b + 2 (t % 8) and the next one: one 16-byte fp16 load per split
// (the partials keep heads in fours, dims consecutive).  Thread t also owns
// head t / 2's (m, l) of every other split, loaded into registers in the same
// round as the partials; the weights then come from independent operations,
// not loops over shared memory (one warp per sub-partition: every latency
// shows).  NS bounds the launch's split count (the loops are unrolled for it).
constexpr int COMB_DIMS = 16;
constexpr int COMB_THREADS = 128;
constexpr int MAX_SPLITS = 64;

template <int NS>
__global__ void __launch_bounds__(COMB_THREADS) combine_tc_kernel(Params p) {
    __shared__ __align__(16) float s_w[MAX_SPLITS][HP];    // split weights
    __shared__ unsigned long long s_live;                  // splits with keys (they wrote a partial)
    __shared__ float s_inv[HP];
    __shared__ int s_bad[HP];
    const int64_t u = blockIdx.x;
    const int dblk = blockIdx.y;
    const int S = p.n_splits;
    const int t = threadIdx.x;
    pdl_wait();                                    // the split partials are complete
    // the first 32 splits' partial rows and this thread's (m, l) pairs cross from L2
    // in one round (an empty split's row holds stale data: it is loaded, never used)
    const int hq = t >> 3;                           // heads 4 hq .. 4 hq + 3
    const int dim = dblk * COMB_DIMS + 2 * (t & 7);  // dims dim, dim + 1
    const uint16_t* po = p.part_o + (static_cast<size_t>(u) * S * HP + 4 * hq) * D + static_cast<size_t>(dim) * 4;
    const size_t split_stride = static_cast<size_t>(HP) * D;
    constexpr int kBatch = NS < 32 ? NS : 32;        // partial loads in flight per thread
    uint4 v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
        v[j] = j < S ? *reinterpret_cast<const uint4*>(po + j * split_stride) : make_uint4(0u, 0u, 0u, 0u);
    const int h = t >> 1, sub = t & 1;               // head h, splits sub, sub + 2, ...
    constexpr int kMl = (NS + 1) / 2;
    const float* ml0 = p.part_ml + static_cast<size_t>(u) * S * 2 * HP;
    float mr[kMl], lr[kMl];
#pragma unroll
    for (int j = 0; j < kMl; ++j) {
        const int sj = sub + 2 * j;
        mr[j] = sj < S ? ml0[sj * 2 * HP + h] : -INFINITY;
        lr[j] = sj < S ? ml0[sj * 2 * HP + HP + h] : 0.0f;
    }
    {
        float M = -INFINITY;
#pragma unroll
        for (int j = 0; j < kMl; ++j)
            if (lr[j] > 0.0f) M = fmaxf(M, mr[j]);
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 1));
        float L = 0.0f;
        int bad = 0;
        unsigned long long live = 0ull;
#pragma unroll
        for (int j = 0; j < kMl; ++j) {
            const int sj = sub + 2 * j;
            if (lr[j] != lr[j]) bad = 1;
            const float wgt = lr[j] > 0.0f ? exp2f(mr[j] - M) * lr[j] : 0.0f;
            if (sj < S) s_w[sj][h] = wgt;
            L += wgt;
            if (lr[j] > 0.0f) live |= 1ull << sj;
        }
        L += __shfl_xor_sync(0xffffffffu, L, 1);
        bad |= __shfl_xor_sync(0xffffffffu, bad, 1);
        // a split holds keys for every head or for none: head 0's view decides
        live |= __shfl_xor_sync(0xffffffffu, live, 1);
        if (t == 0) s_live = live;
        if (sub == 0) {
            // the sink joins the denominator relative to the global max M
            const float sink = p.sink ? __ldg(p.sink + h) : -INFINITY;
            if (p.sink && L > 0.0f) L += exp2f(sink * LOG2E - M);
            s_inv[h] = L > 0.0f ? 1.0f / L : 0.0f;
            s_bad[h] = bad;
            if (p.lse && dblk == 0 && h < p.H)
                p.lse[u * p.H + h] = bad ? __int_as_float(0x7fc00000)
                                         : (L > 0.0f ? (M + log2f(L)) * 0.69314718055994531f : sink);
        }
    }
    __syncthreads();
    const unsigned long long live = s_live;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // [dim offset][head offset]
    for (int s0 = 0; s0 < S; s0 += kBatch) {
        if (s0 > 0) {
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                v[j] = s0 + j < S ? *reinterpret_cast<const uint4*>(po + (s0 + j) * split_stride)
                                  : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int s = s0 + j;
            if (s < S && ((live >> s) & 1ull)) {
                const float4 w4 = *reinterpret_cast<const float4*>(&s_w[s][4 * hq]);
                const float2 a0 = unpack_half2(v[j].x), a1 = unpack_half2(v[j].y);   // dim: heads 0-1, 2-3
                const float2 b0 = unpack_half2(v[j].z), b1 = unpack_half2(v[j].w);   // dim + 1
                acc[0] += w4.x * a0.x; acc[1] += w4.y * a0.y; acc[2] += w4.z * a1.x; acc[3] += w4.w * a1.y;
                acc[4] += w4.x * b0.x; acc[5] += w4.y * b0.y; acc[6] += w4.z * b1.x; acc[7] += w4.w * b1.y;
            }
        }
    }
    const float qnan = __int_as_float(0x7fc00000);
    float cs = 1.0f, sn = 0.0f;
    const bool rot = p.inv_freq && dim >= D - D_ROPE;
    if (rot) rope_cs(p.inv_freq, (dim - (D - D_ROPE)) / 2, unit_pos(p, u), cs, sn);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int h = 4 * hq + i;
        float x = acc[i] * s_inv[h], y = acc[4 + i] * s_inv[h];
        if (rot) {
            // RoPE pair (dim, dim + 1): rotate back by the query's position
            const float x2 = x * cs + y * sn, y2 = y * cs - x * sn;
            x = x2; y = y2;
        }
        if (s_bad[h]) { x = qnan; y = qnan; }
        if (h < p.H) {
            const __nv_bfloat162 o2 = __floats2bfloat162_rn(x, y);
            *reinterpret_cast<__nv_bfloat162*>(p.out + (static_cast<size_t>(u) * p.H + h) * D + dim) = o2;
        }
    }
}

}  // namespace tc

// ---------------------------------------------------------------- host side
namespace {

int launch_tc(tc::Params& p, int64_t units, cudaStream_t st) {
    const bool ex = p.q_norm_w || p.sink || p.inv_freq;
    auto kern = ex ? tc::attn_tc_kernel<true> : tc::attn_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES);
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    // programmatic launches: each kernel waits for its predecessor before any read
    // (but the query, with p.q_early)
    e = launch_pdl(kern, dim3(static_cast<unsigned>(units), p.n_splits), dim3(tc::NTHREADS), tc::SMEM_BYTES, st, p);
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    HCA_CHECK_LAUNCH();
    if (p.n_splits > 1) {
        // the smallest unrolling that covers the split count
        const int S = p.n_splits;
        auto comb = S <= 8 ? tc::combine_tc_kernel<8> : S <= 16 ? tc::combine_tc_kernel<16>
                  : S <= 24 ? tc::combine_tc_kernel<24> : S <= 32 ? tc::combine_tc_kernel<32>
                  : tc::combine_tc_kernel<64>;
        e = launch_pdl(comb, dim3(static_cast<unsigned>(units), tc::D / tc::COMB_DIMS), dim3(tc::COMB_THREADS), 0, st,
                       p);
        if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
        HCA_CHECK_LAUNCH();
    }
    return HCA_OK;
}

}  // namespace

// Split plan of the tensor-core decode path: sparse (CSA) lists favour many
// short splits (latency after top-k); dense (HCA) lists favour a few tiles
// per CTA so the pipeline fills and the partials stay small.
void tc_decode_plan(int B, int max_comp, int W, bool sparse, int& n_splits, int& tiles_per_split) {
    const int n_tiles = static_cast<int>(ceil_div(static_cast<int64_t>(max_comp) + W, tc::TK));
    const int min_tps = sparse ? 1 : 6;       // tiles of 64 keys
    const int budget = launch_budget(sparse ? HCA_BUDGET_SPARSE_DECODE : HCA_BUDGET_DENSE_DECODE);
    int splits = (budget > 0 ? budget : sm_count()) / (B > 0 ? B : 1);
    const int cap_by_len = static_cast<int>(ceil_div(n_tiles > 0 ? n_tiles : 1, min_tps));
    if (splits > cap_by_len) splits = cap_by_len;
    if (splits > tc::MAX_SPLITS) splits = tc::MAX_SPLITS;   // the combine keeps the split weights in shared memory
    if (splits < 1) splits = 1;
    tiles_per_split = static_cast<int>(ceil_div(n_tiles > 0 ? n_tiles : 1, splits));
    n_splits = static_cast<int>(ceil_div(n_tiles > 0 ? n_tiles : 1, tiles_per_split));
}

size_t tc_decode_ws_bytes(int B, int max_comp, int W, bool sparse) {
    int ns, tps;
    tc_decode_plan(B, max_comp, W, sparse, ns, tps);
    if (ns <= 1) return 0;
    // fp16 partial outputs, then fp32 (max, l) pairs
    return static_cast<size_t>(B) * ns * tc::HP * (static_cast<size_t>(tc::D) * 2 + 2 * sizeof(float)) + 256;
}

static void set_extras(tc::Params& p, const hca_attn_extras* ex) {
    if (!ex) return;
    p.q_norm_w = ex->q_norm_w;
    p.norm_eps = ex->norm_eps;
    p.sink = ex->sink;
    p.inv_freq = ex->inv_freq;
    p.q_pos = ex->q_pos;
    p.win_len = ex->win_len;
}

int tc_attn_decode_launch(const uint16_t* q, int B, int H, const hca_kv_cache& kv, const int32_t* idx,
                          int idx_stride, const int32_t* n_comp, int max_comp, const uint16_t* window, int W,
                          float softmax_scale, const hca_attn_extras* ex, uint16_t* out, float* lse, void* ws,
                          size_t ws_bytes, cudaStream_t st) {
    if (B == 0) return HCA_OK;
    tc::Params p = {};
    set_extras(p, ex);
    p.q = q; p.H = H;
    p.codes = kv.codes; p.scales = kv.scales; p.rope = kv.rope; p.cap = kv.capacity;
    p.prefill = 0;
    p.idx = idx; p.idx_stride = idx_stride; p.n_comp = n_comp;
    p.win = window; p.W = W;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    tc_decode_plan(B, max_comp, W, idx != nullptr, p.n_splits, p.tiles_per_split);
    p.q_early = (idx != nullptr && early_query()) ? 1 : 0;
    p.out = out; p.lse = lse;
    if (p.n_splits > 1) {
        const size_t need = tc_decode_ws_bytes(B, max_comp, W, idx != nullptr);
        if (ws == nullptr || ws_bytes < need) return HCA_ERR_WORKSPACE;
        p.part_o = reinterpret_cast<uint16_t*>(ws);
        p.part_ml = reinterpret_cast<float*>(p.part_o + static_cast<size_t>(B) * p.n_splits * tc::HP * tc::D);
    }
    return launch_tc(p, B, st);
}

int tc_attn_prefill_launch(const uint16_t* q, int Tq, int H, int p0, int m, const hca_kv_cache& kv,
                           const int32_t* idx, int idx_stride, const int32_t* count, const uint16_t* raw, int W,
                           float softmax_scale, const hca_attn_extras* ex, uint16_t* out, cudaStream_t st) {
    if (Tq == 0) return HCA_OK;
    tc::Params p = {};
    set_extras(p, ex);
    p.q_pos = nullptr;
    p.win_len = nullptr;
    p.q = q; p.H = H;
    p.codes = kv.codes; p.scales = kv.scales; p.rope = kv.rope; p.cap = kv.capacity;
    p.prefill = 1;
    p.idx = idx; p.idx_stride = idx_stride; p.n_comp = count;
    p.dense_m = m; p.p0 = p0;
    p.win = raw; p.W = W;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.n_splits = 1;
    p.tiles_per_split = 1 << 28;
    p.out = out; p.lse = nullptr;
    return launch_tc(p, Tq, st);
}

// Reads and clears the device error word of the tensor-core attention
// (a bounded wait that gave up).  Synchronous.
int tc_take_device_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_tc_device_error, &z, sizeof(int));
    }
    return v;
}

}  // namespace hca
