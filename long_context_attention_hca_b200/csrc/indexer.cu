// indexer.cu -- lightning indexer scores (CUDA-core path).
//
// "DeepSeek V4: Towards Highly Efficient Million Token Context Intelligence"
// (papers.chlience.com reading note), section 7, the indexer equation
// I_{t,s} = sum_h w^I_{t,h} ReLU(q^I_{t,h} . K^IComp_s), with FP4 operands
// (section 9).  One FP4 e2m1 value times two is a small integer
// (0, +-1, +-2, +-3, +-4, +-6, +-8, +-12), so a 32-element block dot is an
// exact int32 dp4a sum; scaling by the two ue8m0 exponents is exact, and the
// blocks and heads are summed in the fp32 order the C ABI defines.
//
// Work layout: a warp streams NB-lane groups, one lane per 32-element block
// of an entry (NB = c/32), so 8 (c = 128) or 16 (c = 64) entries per warp
// step and a 16-byte load per lane; the query's int8 expansion for the
// lane's block stays in registers for the whole stream.
#include <algorithm>

#include <cuda.h>

#include "common.cuh"

namespace hca {
namespace {

// 8 FP4 codes (one 32-bit word, element 2i in the low nibble of byte i) ->
// 8 int8 values 2*e2m1 in element order (lo word: elements 0..3).
// Byte permutes do the 16-entry table lookup: positive and negative
// magnitude tables, then a per-byte select on the sign bit.
__device__ __forceinline__ void fp4x8_to_i8x8(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t kPos0 = 0x03020100u, kPos1 = 0x0C080604u;     // 0 1 2 3 | 4 6 8 12
    const uint32_t kNeg0 = 0xFDFEFF00u, kNeg1 = 0xF4F8FAFCu;     // -0 -1 -2 -3 | -4 -6 -8 -12
    const uint32_t w_hi = w >> 16;
    {
        const uint32_t s = w & 0x7777u;
        const uint32_t p = __byte_perm(kPos0, kPos1, s);
        const uint32_t n = __byte_perm(kNeg0, kNeg1, s);
        const uint32_t sel = ((w >> 1) & 0x4444u) | 0x3210u;
        lo = __byte_perm(p, n, sel);
    }
    {
        const uint32_t s = w_hi & 0x7777u;
        const uint32_t p = __byte_perm(kPos0, kPos1, s);
        const uint32_t n = __byte_perm(kNeg0, kNeg1, s);
        const uint32_t sel = ((w_hi >> 1) & 0x4444u) | 0x3210u;
        hi = __byte_perm(p, n, sel);
    }
}

// v * 2^e rounded once (round to nearest even), for any integer e: a plain
// product by the exact power of two when 2^e is a normal float, else ldexpf
// (which scales with a single rounding into the subnormal range and to +-inf
// on overflow, and keeps 0 * 2^e = 0 where 2^e itself would overflow).
__device__ __forceinline__ float scale_pow2(float v, int e) {
    if (e >= -126 && e <= 127) return __fmul_rn(v, __uint_as_float(static_cast<uint32_t>(e + 127) << 23));
    return ldexpf(v, e);
}

constexpr int kWarps = 8;
constexpr int kUnroll = 4;   // entries per lane per step, loads issued together

// HI = number of indexer heads (a template bound; Hi <= HI heads are used).
template <int C, int HI>
__global__ void __launch_bounds__(kWarps * 32, HI <= 4 ? 3 : 2)
index_kernel(const uint8_t* __restrict__ q_codes, const uint8_t* __restrict__ q_sf,
             const float* __restrict__ w, const uint8_t* __restrict__ k_codes,
             const uint8_t* __restrict__ k_sf, const int32_t* __restrict__ q_pos,
             int Tq, int64_t Nc_cap, int Hi, int m, int64_t chunk, float* __restrict__ scores) {
    constexpr int NB = C / 32;               // blocks per entry = lanes per entry
    constexpr int EPW = 32 / NB;             // entries per warp per unrolled slot
    constexpr int STEP = EPW * kUnroll;      // entries per warp step
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int blk = lane % NB;
    const int64_t qrow = blockIdx.x;         // b * Tq + t (rows on x: neighbours share a key chunk in L2)
    const int64_t b = qrow / Tq;

    // query expansion for this lane's block, all heads
    uint32_t qv[HI][8];
    int qe[HI];
    float wh[HI];
#pragma unroll
    for (int h = 0; h < HI; ++h) {
        if (h < Hi) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(q_codes + ((qrow * Hi + h) * C / 2) + blk * 16));
            fp4x8_to_i8x8(u.x, qv[h][0], qv[h][1]);
            fp4x8_to_i8x8(u.y, qv[h][2], qv[h][3]);
            fp4x8_to_i8x8(u.z, qv[h][4], qv[h][5]);
            fp4x8_to_i8x8(u.w, qv[h][6], qv[h][7]);
            qe[h] = static_cast<int>(__ldg(q_sf + (qrow * Hi + h) * NB + blk)) - 254;   // eq - 127 + (-127)
            wh[h] = __ldg(w + qrow * Hi + h);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) qv[h][i] = 0;
            qe[h] = 0;
            wh[h] = 0.0f;
        }
    }
    const int64_t pos = q_pos[qrow];
    int64_t elig = (pos + 1) / m;
    elig = elig < 0 ? 0 : (elig > Nc_cap ? Nc_cap : elig);

    const int64_t s_begin = static_cast<int64_t>(blockIdx.y) * chunk;
    const int64_t s_end = min(s_begin + chunk, Nc_cap);
    const int64_t s_live = min(s_end, elig);
    const uint8_t* kc_base = k_codes + static_cast<size_t>(b) * Nc_cap * (C / 2);
    const uint8_t* ks_base = k_sf + static_cast<size_t>(b) * Nc_cap * NB;
    float* out = scores + static_cast<size_t>(qrow) * Nc_cap;

    // ineligible tail of the chunk: -inf, no loads
    for (int64_t s = max(s_begin, elig) + threadIdx.x; s < s_end; s += kWarps * 32) out[s] = -INFINITY;

    for (int64_t s0 = s_begin + warp * STEP; s0 < s_live; s0 += kWarps * STEP) {
        uint4 u[kUnroll];
        int ke[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            const int64_t s = s0 + j * EPW + lane / NB;
            if (s < s_live) {
                u[j] = __ldg(reinterpret_cast<const uint4*>(kc_base + s * (C / 2) + blk * 16));
                ke[j] = static_cast<int>(__ldg(ks_base + s * NB + blk));
            } else {
                u[j] = make_uint4(0, 0, 0, 0);
                ke[j] = 0;
            }
        }
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            const int64_t s = s0 + j * EPW + lane / NB;
            uint32_t kv[8];
            fp4x8_to_i8x8(u[j].x, kv[0], kv[1]);
            fp4x8_to_i8x8(u[j].y, kv[2], kv[3]);
            fp4x8_to_i8x8(u[j].z, kv[4], kv[5]);
            fp4x8_to_i8x8(u[j].w, kv[6], kv[7]);
            float dot[HI];
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                int acc = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc = __dp4a(static_cast<int>(kv[i]), static_cast<int>(qv[h][i]), acc);
                // block dot = acc / 4 exactly; times 2^(eq + ek - 254)
                const float t = scale_pow2(static_cast<float>(acc), qe[h] + ke[j] - 2);
                // ordered block sum on the entry's first lane: ((t0 + t1) + t2) + t3
                float a = t;
#pragma unroll
                for (int q = 1; q < NB; ++q) a = __fadd_rn(a, __shfl_down_sync(0xffffffffu, t, q));
                dot[h] = a;
            }
            if (blk == 0 && s < s_live) {
                float sc = 0.0f;
#pragma unroll
                for (int h = 0; h < HI; ++h) {
                    if (h < Hi) {
                        const float r = dot[h] > 0.0f ? dot[h] : 0.0f;
                        sc = __fadd_rn(sc, __fmul_rn(wh[h], r));
                    }
                }
                out[s] = sc;
            }
        }
    }
}

// ------------------------------------------------------------------ tensor-pipe path (c = 128, Hi = 4)
// 8 FP4 codes of one 32-bit word -> 4 f16x2 words (hardware e2m1 -> f16,
// exact).  Keys and queries go through this same conversion, so the pairing
// of elements in every product is the same whichever nibble lands in which
// half.
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2, uint32_t& o3) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3) : "r"(w));
}

__device__ __forceinline__ void hmma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One warp scores 16 entries per m16n8k16 tile.  Lane (g = lane/4, q = lane%4)
// loads bytes 16q..16q+15 (block q, elements 32q..32q+31) of rows g and
// g+8; k-step s, columns 2q+e and 8+2q+e hold elements 32q+4s+e and
// 32q+4s+2+e.  The 16 output columns are (block b, head h) pairs, two blocks
// per n-tile; the query operand is the head's values where the element's
// block equals the column's block and zero elsewhere, so each column is one
// exact 32-element block dot.
constexpr int kMmaWarps = 8;
constexpr int kAhead = 2;        // tiles of raw keys in flight per warp beyond the current one

__global__ void __launch_bounds__(kMmaWarps * 32, 2)
index_mma_kernel(const uint8_t* __restrict__ q_codes, const uint8_t* __restrict__ q_sf,
                 const float* __restrict__ w, const uint8_t* __restrict__ k_codes,
                 const uint8_t* __restrict__ k_sf, const int32_t* __restrict__ q_pos,
                 int Tq, int64_t Nc_cap, int m, int64_t chunk, float* __restrict__ scores) {
    constexpr int C = 128, HI = 4;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int64_t qrow = blockIdx.x;
    const int64_t b = qrow / Tq;

    // query operand: n-tile nt covers blocks 2nt, 2nt+1; this lane's column n = g
    uint32_t bq[2][8][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int blk = 2 * nt + (g >> 2), h = g & 3;
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(q_codes + (qrow * HI + h) * (C / 2) + q * 16));
        uint32_t Q[16];
        e2m1x8_to_f16x8(u.x, Q[0], Q[1], Q[2], Q[3]);
        e2m1x8_to_f16x8(u.y, Q[4], Q[5], Q[6], Q[7]);
        e2m1x8_to_f16x8(u.z, Q[8], Q[9], Q[10], Q[11]);
        e2m1x8_to_f16x8(u.w, Q[12], Q[13], Q[14], Q[15]);
        const bool on = (q == blk);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            bq[nt][s][0] = on ? Q[2 * s] : 0u;
            bq[nt][s][1] = on ? Q[2 * s + 1] : 0u;
        }
    }
    // scale exponents of the accumulator columns this lane holds:
    // n-tile nt, j in {0,1}: block 2nt + q/2, head 2(q%2) + j
    int eqv[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j)
            eqv[nt][j] = static_cast<int>(__ldg(q_sf + (qrow * HI + 2 * (q & 1) + j) * 4 + 2 * nt + (q >> 1))) - 254;
    float wh[HI];
#pragma unroll
    for (int h = 0; h < HI; ++h) wh[h] = __ldg(w + qrow * HI + h);

    const int64_t pos = q_pos[qrow];
    int64_t elig = (pos + 1) / m;
    elig = elig < 0 ? 0 : (elig > Nc_cap ? Nc_cap : elig);
    const int64_t s_begin = static_cast<int64_t>(blockIdx.y) * chunk;
    const int64_t s_end = min(s_begin + chunk, Nc_cap);
    const int64_t s_live = min(s_end, elig);
    const uint8_t* kc_base = k_codes + static_cast<size_t>(b) * Nc_cap * (C / 2);
    const uint32_t* ks_base = reinterpret_cast<const uint32_t*>(k_sf + static_cast<size_t>(b) * Nc_cap * 4);
    float* out = scores + static_cast<size_t>(qrow) * Nc_cap;

    for (int64_t s = max(s_begin, elig) + threadIdx.x; s < s_end; s += kMmaWarps * 32) out[s] = -INFINITY;

    const int64_t n_tiles = s_live > s_begin ? (s_live - s_begin + 15) / 16 : 0;
    // raw-key ring: tiles t, t+kMmaWarps, ... of this warp
    uint4 rk[kAhead + 1][2];
    uint32_t rs[kAhead + 1][2];
    auto fetch = [&](int64_t tile, int slot) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int64_t e = s_begin + tile * 16 + g + 8 * r;
            if (tile < n_tiles && e < s_live) {
                rk[slot][r] = __ldg(reinterpret_cast<const uint4*>(kc_base + e * (C / 2) + q * 16));
                rs[slot][r] = __ldg(ks_base + e);
            } else {
                rk[slot][r] = make_uint4(0, 0, 0, 0);
                rs[slot][r] = 0x7F7F7F7Fu;
            }
        }
    };
#pragma unroll
    for (int a = 0; a < kAhead; ++a) fetch(warp + static_cast<int64_t>(a) * kMmaWarps, a);
    constexpr int slot = 0;                      // the ring rotates, so the current tile is always slot 0
    for (int64_t tile = warp; tile < n_tiles; tile += kMmaWarps) {
        fetch(tile + static_cast<int64_t>(kAhead) * kMmaWarps, kAhead);
        uint32_t A0[16], A1[16];
        {
            const uint4 u0 = rk[slot][0], u1 = rk[slot][1];
            e2m1x8_to_f16x8(u0.x, A0[0], A0[1], A0[2], A0[3]);
            e2m1x8_to_f16x8(u0.y, A0[4], A0[5], A0[6], A0[7]);
            e2m1x8_to_f16x8(u0.z, A0[8], A0[9], A0[10], A0[11]);
            e2m1x8_to_f16x8(u0.w, A0[12], A0[13], A0[14], A0[15]);
            e2m1x8_to_f16x8(u1.x, A1[0], A1[1], A1[2], A1[3]);
            e2m1x8_to_f16x8(u1.y, A1[4], A1[5], A1[6], A1[7]);
            e2m1x8_to_f16x8(u1.z, A1[8], A1[9], A1[10], A1[11]);
            e2m1x8_to_f16x8(u1.w, A1[12], A1[13], A1[14], A1[15]);
        }
        float D0[4] = {0.f, 0.f, 0.f, 0.f}, D1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            hmma16816(D0, A0[2 * s], A1[2 * s], A0[2 * s + 1], A1[2 * s + 1], bq[0][s][0], bq[0][s][1]);
            hmma16816(D1, A0[2 * s], A1[2 * s], A0[2 * s + 1], A1[2 * s + 1], bq[1][s][0], bq[1][s][1]);
        }
        // scale: D0 = block q/2, D1 = block 2 + q/2; [j + 2r] = head 2(q%2)+j, row g + 8r
        float tA[2][2], tB[2][2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t sw = rs[slot][r];
            const int ekA = static_cast<int>((sw >> (8 * (q >> 1))) & 0xFFu);
            const int ekB = static_cast<int>((sw >> (8 * (2 + (q >> 1)))) & 0xFFu);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                tA[j][r] = scale_pow2(D0[j + 2 * r], eqv[0][j] + ekA);
                tB[j][r] = scale_pow2(D1[j + 2 * r], eqv[1][j] + ekB);
            }
        }
        // lanes q = 0, 1 hold blocks 0 and 2; lanes q = 2, 3 blocks 1 and 3 (same heads as q - 2)
        float dot[2][2];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float t1 = __shfl_down_sync(0xffffffffu, tA[j][r], 2);
                const float t3 = __shfl_down_sync(0xffffffffu, tB[j][r], 2);
                dot[j][r] = __fadd_rn(__fadd_rn(__fadd_rn(tA[j][r], t1), tB[j][r]), t3);
            }
        // lane q = 0 holds heads 0, 1; lane q = 1 heads 2, 3
        float hi2[2][2];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int r = 0; r < 2; ++r) hi2[j][r] = __shfl_down_sync(0xffffffffu, dot[j][r], 1);
        if (q == 0) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int64_t e = s_begin + tile * 16 + g + 8 * r;
                if (e < s_live) {
                    const float d4[4] = {dot[0][r], dot[1][r], hi2[0][r], hi2[1][r]};
                    float sc = 0.0f;
#pragma unroll
                    for (int h = 0; h < HI; ++h) sc = __fadd_rn(sc, __fmul_rn(wh[h], d4[h] > 0.0f ? d4[h] : 0.0f));
                    out[e] = sc;
                }
            }
        }
#pragma unroll
        for (int a = 0; a < kAhead; ++a) {
            rk[a][0] = rk[a + 1][0]; rk[a][1] = rk[a + 1][1];
            rs[a][0] = rs[a + 1][0]; rs[a][1] = rs[a + 1][1];
        }
    }
}

// ------------------------------------------------------------------ tcgen05 path (c = 128, Hi = 4)
// The tensor cores read FP4 e2m1 operands straight from shared memory
// (tcgen05.mma kind::f8f6f4, fp32 accumulation), laid out as 16-element
// groups in 16-byte slots (8 data bytes, then 8 bytes of padding) in the
// K-major 128-byte-swizzled layout.  The key tiles arrive in exactly that
// layout from the tensor memory accelerator: a tensor map of type
// 16U4_ALIGN16B spreads 64 packed bytes per key over a 128-byte row.  It
// writes only the data bytes (the padding is zeroed once per CTA) and its
// transaction count is the packed size, 64 bytes per key.
// A = 128 keys (one per TMEM lane), B = 16 columns per query: column
// (block b, head h) holds head h's values on block b's 32 elements and zeros
// elsewhere, so every accumulator column is one exact 32-element block dot.
// The thread that owns a TMEM lane (one key) applies the two ue8m0 exponents
// exactly and sums blocks and heads in the order the C ABI defines.
//
// Warp roles: warp 0 issues the tensor-map loads of key codes and key scales
// into a ring of KS stages, warp 1 issues the MMAs into NBD accumulator
// buffers, warps 2.. run the epilogue (EG warps per TMEM lane quarter, each
// taking every EG-th query).  Every wait is bounded; a wait that gives up
// raises the device error word and the scores of that CTA become NaN.
namespace itc {

constexpr int TILE = 128;                    // keys per tile (MMA M)
constexpr int CODE_BYTES = TILE * 128;       // 16 KB of unpacked FP4 per tile
constexpr int CODE_TX_BYTES = TILE * 64;     // the load's transaction count: packed bytes read
constexpr int SCALE_BYTES = TILE * 4;        // ue8m0 x 4 per key
constexpr int STAGE_BYTES = CODE_BYTES + 1024;
constexpr long long kWaitLimit = 1ll << 24;

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
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void tma_load_1d(uint32_t dst, const CUtensorMap* map, int x, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2}], [%3];"
                 :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(bar) : "memory");
}
__device__ __forceinline__ uint64_t sdesc(uint32_t addr) {   // K-major SW128, 8-row groups 1024 B apart
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ uint32_t sw128(int row, int slot) {
    return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((slot ^ (row & 7)) << 4));
}

__device__ int g_index_device_error = 0;    // a bounded wait gave up (outputs are NaN)

// bounded wait; on give-up raise the CTA's abort flag and the device error word
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    for (long long it = 0; it < kWaitLimit; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 1023) == 1023 && *abort_flag) return false;
    }
    *abort_flag = 1;
    atomicExch(&g_index_device_error, 1);
    return false;
}

// The same wait for the single-thread roles (loads, MMA issue), with a short
// sleep between polls: their spinning would otherwise take issue slots from the
// epilogue warps that share their sub-partitions.
__device__ __forceinline__ bool wait_bar_idle(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    for (long long it = 0; it < kWaitLimit; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        __nanosleep(32);
        if ((it & 1023) == 1023 && *abort_flag) return false;
    }
    *abort_flag = 1;
    atomicExch(&g_index_device_error, 1);
    return false;
}

// QG queries per CTA, HG groups of 4 indexer heads (Hi = 4 HG; N = 16 QG HG
// accumulator columns: query q, group hg at column 16 (q HG + hg), then block
// b, head h of the group at + 4 b + h), NBD accumulator buffers, KS key
// stages, EG epilogue warps per TMEM lane quarter.  bf16: the scores are
// written rounded to bf16 (nearest even) as uint16 bit patterns, and the
// histogram counts the rounded values.
// Larger key = larger score; +0 and -0 map to the same key (the top-k's order).
__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// hist (optional, one query per CTA): the query row's 2048-bin histogram of the
// top 11 bits of each eligible score's key, hist + row * hist_stride (u32),
// accumulated in shared memory and added with global atomics at the end.
template <int QG, int NBD, int KS, int EG, int HG>
__global__ void __launch_bounds__(64 + 128 * EG)
index_tc_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales,
                const uint8_t* __restrict__ q_codes, const uint8_t* __restrict__ q_sf,
                const float* __restrict__ w, const int32_t* __restrict__ q_pos,
                int Tq, int64_t Nc_cap, int m, int64_t chunk, float* __restrict__ scores,
                uint32_t* __restrict__ hist, int64_t hist_stride, int bf16) {
    constexpr int HI = 4 * HG;
    constexpr int N = 16 * QG * HG;
    constexpr uint32_t NCOLS = (N * NBD) <= 32 ? 32 : (N * NBD <= 64 ? 64 : (N * NBD <= 128 ? 128 : (N * NBD <= 256 ? 256 : 512)));
    constexpr uint32_t IDESC = (1u << 4) | (5u << 7) | (5u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
                               (static_cast<uint32_t>(TILE >> 4) << 24);
    constexpr int EPI = 4 * EG;                         // epilogue warps
    pdl_trigger();                                      // the top-k select may be placed early (it waits)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sB = smem + KS * STAGE_BYTES;              // N rows x 128 B (query operand)
    uint32_t* sh_hist = reinterpret_cast<uint32_t*>(sB + N * 128);   // 2048 bins when hist != nullptr
    __shared__ __align__(8) uint64_t bar_full[KS], bar_empty[KS], bar_accf[NBD], bar_acce[NBD], bar_drain;
    __shared__ uint32_t tmem_slot;
    __shared__ int s_eq[QG][16 * HG];                   // (uq - 127) - 127 per (query, group*16 + block*4 + head)
    __shared__ __align__(16) int s_klo[QG][HG][4];      // key exponent range of the fast path per (group, block)
    __shared__ __align__(16) int s_khi[QG][HG][4];
    __shared__ __align__(16) float s_qf[QG][16 * HG];   // 2^(uq - 127) per (query, group*16 + block*4 + head)
    __shared__ float s_w[QG][HI];
    uint16_t* scores16 = reinterpret_cast<uint16_t*>(scores);
    __shared__ int64_t s_elig[QG];
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t qrow0 = static_cast<int64_t>(blockIdx.x) * QG;     // first query row (b * Tq + t)
    const int64_t b = qrow0 / Tq;                                    // all QG rows share a sequence
    const int64_t s_begin = static_cast<int64_t>(blockIdx.y) * chunk;
    const int64_t s_end = min(s_begin + chunk, Nc_cap);

    if (tid == 0) {
        // warps that release a tile: all epilogue warps, or (one query per CTA) the 4 of the tile's group
        constexpr int REL = QG == 1 ? 4 : EPI;
        for (int i = 0; i < KS; ++i) { mbar_init(smem_u32(&bar_full[i]), 1); mbar_init(smem_u32(&bar_empty[i]), REL); }
        for (int i = 0; i < NBD; ++i) { mbar_init(smem_u32(&bar_accf[i]), 1); mbar_init(smem_u32(&bar_acce[i]), REL); }
        mbar_init(smem_u32(&bar_drain), 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(smem_u32(&tmem_slot)), "r"(NCOLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // the query's operands and exponents: every global load of the prologue is issued
    // before any of them is used (one round trip, not one per table)
    constexpr int NQV = N * 8;                          // 16-byte slots of the query operand
    constexpr int QV_PT = (NQV + (64 + 128 * EG) - 1) / (64 + 128 * EG);
    uint2 qv[QV_PT];
#pragma unroll
    for (int k2 = 0; k2 < QV_PT; ++k2) {
        const int x = tid + k2 * blockDim.x;
        qv[k2] = make_uint2(0u, 0u);
        if (x < NQV) {
            const int n = x >> 3, j = x & 7;
            const int q = n / (16 * HG), blk = (n >> 2) & 3, h = ((n >> 4) % HG) * 4 + (n & 3);
            if ((j >> 1) == blk) qv[k2] = __ldg(reinterpret_cast<const uint2*>(q_codes + ((qrow0 + q) * HI + h) * 64 + j * 8));
        }
    }
    // exponents of (query, group hg, block blk, head hh) at z = hg 16 + blk 4 + hh
    static_assert(QG * 16 * HG <= 64 + 128 * EG && QG * HI <= 64 + 128 * EG, "one exponent and weight per thread");
    const bool has_e = tid < QG * 16 * HG;
    int e_raw = 0;
    if (has_e) {
        const int q = tid / (16 * HG), z = tid % (16 * HG), hg = z >> 4, blk = (z >> 2) & 3, h = hg * 4 + (z & 3);
        e_raw = static_cast<int>(__ldg(q_sf + ((qrow0 + q) * HI + h) * 4 + blk)) - 254;
    }
    const float w_raw = tid < QG * HI ? __ldg(w + (qrow0 + tid / HI) * HI + tid % HI) : 0.0f;
    const int32_t pos_raw = tid < QG ? q_pos[qrow0 + tid] : 0;
    if (QG == 1 && hist)
        for (int x = tid; x < 2048; x += blockDim.x) sh_hist[x] = 0u;
    // the loads write only the 8 data bytes of each 16-byte slot: zero the padding once
    for (int x = tid; x < KS * (CODE_BYTES / 16); x += blockDim.x) {
        const int st = x / (CODE_BYTES / 16), o = x % (CODE_BYTES / 16);
        *reinterpret_cast<uint4*>(smem + st * STAGE_BYTES + o * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    // query operand: row n = (q HG + hg) 16 + blk 4 + hh (head h = 4 hg + hh); slot j
    // (elements 16j..16j+15) is block j/2
#pragma unroll
    for (int k2 = 0; k2 < QV_PT; ++k2) {
        const int x = tid + k2 * blockDim.x;
        if (x < NQV) *reinterpret_cast<uint4*>(sB + sw128(x >> 3, x & 7)) = make_uint4(qv[k2].x, qv[k2].y, 0u, 0u);
    }
    if (has_e) s_eq[tid / (16 * HG)][tid % (16 * HG)] = e_raw;
    if (tid < QG * HI) s_w[tid / HI][tid % HI] = w_raw;
    if (tid < QG) {
        const int64_t e = (static_cast<int64_t>(pos_raw) + 1) / m;
        s_elig[tid] = e < 0 ? 0 : (e > Nc_cap ? Nc_cap : e);
    }
    __syncthreads();
    for (int x = tid; x < QG * HG * 4; x += blockDim.x) {
        // fast path of a (query, group, block): every head's 2^(eq + ek) is a normal float and
        // |block dot| * 2^(eq + ek) < 2^127, i.e. eq + ek in [-126, 116] for the group's heads
        const int q = x / (HG * 4), hg = (x / 4) % HG, blk = x & 3;
        int mn = 1 << 20, mx = -(1 << 20);
        for (int hh = 0; hh < 4; ++hh) {
            const int e = s_eq[q][hg * 16 + blk * 4 + hh];
            mn = min(mn, e);
            mx = max(mx, e);
        }
        int lo = -126 - mn, hi = 116 - mx;
        if (!(QG == 1 && HG == 1)) {
            // the fast path of this instantiation takes each term as (D * 2^(uq - 127)) *
            // 2^(uk - 127): the key factor a normal float (uk in [1, 254]) and the first
            // product exact for every block dot (|D| in [1/4, 1152] or 0): uq in [3, 244]
            lo = max(lo, 1);
            hi = min(hi, 254);
            if (mn + 254 < 3 || mx + 254 > 244) { lo = 1; hi = 0; }
        }
        s_klo[q][hg][blk] = lo;
        s_khi[q][hg][blk] = hi;
    }
    for (int x = tid; x < QG * HG * 16; x += blockDim.x) {
        const int uq = s_eq[x / (16 * HG)][x % (16 * HG)] + 254;
        s_qf[x / (16 * HG)][x % (16 * HG)] = (uq >= 1 && uq <= 254) ? __uint_as_float(static_cast<uint32_t>(uq) << 23) : 0.0f;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_slot;
    int64_t elig_max = 0;
    for (int q = 0; q < QG; ++q) elig_max = max(elig_max, s_elig[q]);
    const int64_t s_live = min(s_end, elig_max);
    const int n_tiles = s_live > s_begin ? static_cast<int>((s_live - s_begin + TILE - 1) / TILE) : 0;

    // ineligible part of the chunk: -inf (per query)
    for (int q = 0; q < QG; ++q) {
        const size_t ro = static_cast<size_t>(qrow0 + q) * Nc_cap;
        for (int64_t s = max(s_begin, s_elig[q]) + tid; s < s_end; s += blockDim.x) {
            if (bf16) scores16[ro + s] = 0xFF80u;
            else scores[ro + s] = -INFINITY;
        }
    }
    const int row0 = static_cast<int>(b * Nc_cap + s_begin);        // tensor-map row of the chunk's first key

    if (warp == 0) {
        // ---------------------------------------------------------------- loads
        if (lane == 0) {
            for (int t = 0; t < n_tiles; ++t) {
                const int st = t % KS;
                if (t >= KS && !wait_bar_idle(smem_u32(&bar_empty[st]), ((t / KS) - 1) & 1, &s_abort)) break;
                const uint32_t full = smem_u32(&bar_full[st]);
                uint8_t* stage = smem + st * STAGE_BYTES;
                mbar_expect_tx(full, CODE_TX_BYTES + SCALE_BYTES);
                tma_load_2d(smem_u32(stage), &tm_codes, 0, row0 + t * TILE, full);
                tma_load_1d(smem_u32(stage + CODE_BYTES), &tm_scales, row0 + t * TILE, full);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t bbase = smem_u32(sB);
            for (int t = 0; t < n_tiles; ++t) {
                const int st = t % KS, nb = t % NBD;
                if (!wait_bar_idle(smem_u32(&bar_full[st]), (t / KS) & 1, &s_abort)) break;
                if (t >= NBD && !wait_bar_idle(smem_u32(&bar_acce[nb]), ((t / NBD) - 1) & 1, &s_abort)) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t abase = smem_u32(smem + st * STAGE_BYTES);
                const uint32_t d = tmem + static_cast<uint32_t>(nb * N);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                 "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                                 :: "r"(d), "l"(sdesc(abase + kk * 32)), "l"(sdesc(bbase + kk * 32)), "r"(IDESC), "r"(kk)
                                 : "memory");
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                             :: "r"(smem_u32(&bar_accf[nb])) : "memory");
            }
            // completes once every MMA issued above has finished
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         :: "r"(smem_u32(&bar_drain)) : "memory");
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        // items i = (tile t, j-th query of this warp), in order; the TMEM load of item
        // i + 1 is in flight while item i is scored
        // one query per CTA: the EG warps of a lane quarter take alternate tiles; else
        // they split the queries of every tile
        constexpr int QPW = QG == 1 ? 1 : QG / EG;     // queries per epilogue warp and tile
        constexpr int TS = QG == 1 ? EG : 1;           // tile stride
        constexpr int QE = QG == 1 ? 1 : EG;           // query stride
        const int quarter = warp & 3;                  // TMEM lanes 32 quarter .. +31
        const int eg = (warp - 2) >> 2;                // this warp's share of the tiles or queries
        const int t0 = QG == 1 ? eg : 0, q0 = QG == 1 ? 0 : eg;
        const int row = quarter * 32 + lane;           // key row of the tile
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const int n_mine = n_tiles > t0 ? (n_tiles - t0 + TS - 1) / TS : 0;
        const int n_items = n_mine * QPW;
        // sub-items I = (item i, chunk ch of GPC head groups): the TMEM loads of sub-item
        // I + 1 are in flight while I is scored; a score is complete after its last chunk
        constexpr int GPC = HG >= 4 ? 4 : HG;          // head groups per chunk (16 columns each)
        constexpr int NCH = HG / GPC;                   // chunks per item
        const int n_sub = n_items * NCH;
        int eq1[16], klo1[4], khi1[4];                 // the only query's exponents (QG == 1, HG == 1)
#pragma unroll
        for (int j = 0; j < 16; ++j) eq1[j] = s_eq[0][j];
#pragma unroll
        for (int j = 0; j < 4; ++j) { klo1[j] = s_klo[0][0][j]; khi1[j] = s_khi[0][0][j]; }
        uint32_t rn[16 * GPC];
        auto tmem_ld = [&](int I) {
            const int i = I / NCH, ch = I % NCH;
            const int t = t0 + TS * (i / QPW), q = q0 + QE * (i % QPW);
#pragma unroll
            for (int g = 0; g < GPC; ++g) {
                uint32_t* d = rn + 16 * g;
                asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                             : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]), "=r"(d[7]),
                               "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
                             : "r"(lane_base + static_cast<uint32_t>((t % NBD) * N + (q * HG + ch * GPC + g) * 16)));
            }
        };
        // a tile's accumulators are complete (and its stage's loads visible) after these waits
        auto tile_ready = [&](int t) {
            if (!wait_bar(smem_u32(&bar_accf[t % NBD]), (t / NBD) & 1, &s_abort)) return false;
            if (!wait_bar(smem_u32(&bar_full[t % KS]), (t / KS) & 1, &s_abort)) return false;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            return true;
        };
        bool ok = true;
        if (n_sub > 0) {
            if (tile_ready(t0)) tmem_ld(0); else ok = false;
        }
        uint32_t sw = 0;
        float sc = 0.0f;
        for (int I = 0; I < n_sub && ok; ++I) {
            const int i = I / NCH, ch = I % NCH;
            const int t = t0 + TS * (i / QPW), j = i % QPW, q = q0 + QE * j;
            const int st = t % KS, nb = t % NBD;
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            uint32_t rc[16 * GPC];
#pragma unroll
            for (int z = 0; z < 16 * GPC; ++z) rc[z] = rn[z];
            if (j == 0 && ch == 0) sw = *reinterpret_cast<const uint32_t*>(smem + st * STAGE_BYTES + CODE_BYTES + row * 4);
            if (j == QPW - 1 && ch == NCH - 1) {
                // every load of tile t has completed and its scale word is read: release
                // the accumulator buffer and the key stage
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) { mbar_arrive(smem_u32(&bar_acce[nb])); mbar_arrive(smem_u32(&bar_empty[st])); }
            }
            if (I + 1 < n_sub) {
                if ((I + 1) % (QPW * NCH) == 0 && !tile_ready(t + TS)) { ok = false; }
                else tmem_ld(I + 1);
            }
#pragma unroll
            for (int g = 0; g < GPC; ++g) {
            const int hg = ch * GPC + g;
            const uint32_t* r = rc + 16 * g;
            constexpr bool kOne = QG == 1 && HG == 1;
            int ek[4];
            bool fast = true;
            int4 lo4 = make_int4(0, 0, 0, 0), hi4 = make_int4(0, 0, 0, 0);
            if (!kOne) {
                lo4 = *reinterpret_cast<const int4*>(&s_klo[q][hg][0]);
                hi4 = *reinterpret_cast<const int4*>(&s_khi[q][hg][0]);
            }
            const int los[4] = {lo4.x, lo4.y, lo4.z, lo4.w}, his[4] = {hi4.x, hi4.y, hi4.z, hi4.w};
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                ek[blk] = static_cast<int>((sw >> (8 * blk)) & 0xFFu);
                const int lo = kOne ? klo1[blk] : los[blk];
                const int hi = kOne ? khi1[blk] : his[blk];
                fast &= (ek[blk] >= lo) & (ek[blk] <= hi);
            }
            float dot[4];
            if (__all_sync(0xffffffffu, fast)) {
                // every term is an exact product (a normal power of two, no overflow), so
                // fma(D, 2^e, acc) rounds exactly as the ordered sum acc + D * 2^e does
                if (kOne) {
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
#pragma unroll
                        for (int blk = 0; blk < 4; ++blk) {
                            const int z = blk * 4 + h;
                            const float s2 = __uint_as_float(static_cast<uint32_t>(eq1[z] + 127 + ek[blk]) << 23);
                            dot[h] = blk == 0 ? __fmul_rn(__uint_as_float(r[z]), s2)
                                              : __fmaf_rn(__uint_as_float(r[z]), s2, dot[h]);
                        }
                    }
                } else {
                    // D * 2^(eq + ek) as (D * 2^(uq - 127)) * 2^(uk - 127): the first product is
                    // exact (the range above), so the fma's single rounding is the same one
                    float qf[16];
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float4 f = *reinterpret_cast<const float4*>(&s_qf[q][hg * 16 + 4 * v]);
                        qf[4 * v] = f.x; qf[4 * v + 1] = f.y; qf[4 * v + 2] = f.z; qf[4 * v + 3] = f.w;
                    }
                    float kf[4];
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) kf[blk] = __uint_as_float(static_cast<uint32_t>(ek[blk]) << 23);
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
#pragma unroll
                        for (int blk = 0; blk < 4; ++blk) {
                            const int z = blk * 4 + h;
                            const float a = __fmul_rn(__uint_as_float(r[z]), qf[z]);
                            dot[h] = blk == 0 ? __fmul_rn(a, kf[blk]) : __fmaf_rn(a, kf[blk], dot[h]);
                        }
                    }
                }
            } else {
                int eq[16];
#pragma unroll
                for (int z = 0; z < 16; ++z) eq[z] = kOne ? eq1[z] : s_eq[q][hg * 16 + z];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    // column blk*4 + h: ordered block sum ((t0 + t1) + t2) + t3, each term rounded once
                    float a = scale_pow2(__uint_as_float(r[h]), eq[h] + ek[0]);
#pragma unroll
                    for (int blk = 1; blk < 4; ++blk)
                        a = __fadd_rn(a, scale_pow2(__uint_as_float(r[blk * 4 + h]), eq[blk * 4 + h] + ek[blk]));
                    dot[h] = a;
                }
            }
            // heads 4 hg .. 4 hg + 3, continuing the ordered sum over h = 0 .. Hi - 1
            if (hg == 0) sc = 0.0f;
#pragma unroll
            for (int h = 0; h < 4; ++h)
                sc = __fadd_rn(sc, __fmul_rn(s_w[q][hg * 4 + h], dot[h] > 0.0f ? dot[h] : 0.0f));
            if (hg == HG - 1) {
                const int64_t e = s_begin + static_cast<int64_t>(t) * TILE + row;
                if (e < s_end && e < s_elig[q]) {
                    const size_t o = static_cast<size_t>(qrow0 + q) * Nc_cap + e;
                    if (bf16) {
                        const uint16_t hb = ok ? __bfloat16_as_ushort(__float2bfloat16_rn(sc)) : 0x7FC0u;
                        scores16[o] = hb;
                        if (QG == 1 && hist && ok)
                            atomicAdd(&sh_hist[score_key(__uint_as_float(static_cast<uint32_t>(hb) << 16)) >> 21], 1u);
                    } else {
                        scores[o] = ok ? sc : __int_as_float(0x7fc00000);
                        // a NaN score is not counted: after a device error the top-k is undefined anyway
                        if (QG == 1 && hist && ok) atomicAdd(&sh_hist[score_key(sc) >> 21], 1u);
                    }
                }
            }
            }   // head groups of the chunk
        }
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (!ok) {
            // scores of the tiles this warp did not reach: NaN
            for (int q = q0; q < QG; q += QE)
                for (int64_t e = s_begin + row; e < s_live; e += TILE)
                    if (e < s_elig[q]) {
                        const size_t o = static_cast<size_t>(qrow0 + q) * Nc_cap + e;
                        if (bf16) scores16[o] = 0x7FC0u;
                        else scores[o] = __int_as_float(0x7fc00000);
                    }
        }
    }
    __syncthreads();
    if (QG == 1 && hist) {
        uint32_t* gh = hist + qrow0 * hist_stride;
        for (int x = tid; x < 2048; x += blockDim.x) {
            const uint32_t v = sh_hist[x];
            if (v) atomicAdd(&gh[x], v);
        }
    }
    if (warp == 1) {
        // no MMA may still write TMEM when it is released
        if (lane == 0) wait_bar(smem_u32(&bar_drain), 0, &s_abort);
        __syncwarp();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(NCOLS) : "memory");
    }
}

// tensor maps of the keys: codes as [rows][128] 4-bit values (64 B a row,
// unpacked to 128 B a row in shared memory), scales as [rows] 32-bit words
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// false when the key buffers do not meet the tensor-map rules (the caller
// then takes the CUDA-core path)
bool make_maps(const uint8_t* k_codes, const uint8_t* k_sf, int64_t rows, int64_t nc_cap, CUtensorMap* codes,
               CUtensorMap* scales) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if ((reinterpret_cast<uintptr_t>(k_codes) & 31u) || (reinterpret_cast<uintptr_t>(k_sf) & 15u)) return false;
    if (rows <= 0 || rows > 0x7FFFFFFFLL) return false;
    // a tile's scale words start at x = row (32-bit elements): x * 4 must be a
    // multiple of 16 bytes, so every sequence must start on a multiple of 4 rows
    if (nc_cap % 4 != 0) return false;
    const cuuint64_t cdim[2] = {128, static_cast<cuuint64_t>(rows)};
    const cuuint64_t cstride[1] = {64};
    const cuuint32_t cbox[2] = {128, TILE};
    const cuuint32_t ones[2] = {1, 1};
    if (fn(codes, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<uint8_t*>(k_codes), cdim, cstride, cbox, ones,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    const cuuint64_t sdim[1] = {static_cast<cuuint64_t>(rows)};
    const cuuint64_t sstride[1] = {4};   // unused at rank 1
    const cuuint32_t sbox[1] = {TILE};
    if (fn(scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 1, const_cast<uint8_t*>(k_sf), sdim, sstride, sbox, ones,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    return true;
}

// returns HCA_ERR_UNSUPPORTED (nothing launched) when the tensor maps cannot be made
template <int QG, int NBD, int KS, int EG, int HG = 1>
int launch_tc(const uint8_t* q_codes, const uint8_t* q_sf, const float* w, const uint8_t* k_codes,
              const uint8_t* k_sf, const int32_t* q_pos, int64_t rows, int B, int Tq, int64_t Nc_cap, int m,
              float* scores, cudaStream_t st, int64_t want_ctas, uint32_t* hist = nullptr, int64_t hist_stride = 0,
              int bf16 = 0) {
    CUtensorMap tm_codes, tm_scales;
    if (!make_maps(k_codes, k_sf, static_cast<int64_t>(B) * Nc_cap, Nc_cap, &tm_codes, &tm_scales)) return HCA_ERR_UNSUPPORTED;
    const int64_t groups = rows / QG;
    int64_t chunk = ceil_div(Nc_cap, std::max<int64_t>(1, want_ctas / std::max<int64_t>(groups, 1)));
    chunk = ceil_div(chunk, TILE) * TILE;
    if (chunk < TILE) chunk = TILE;
    if (ceil_div(Nc_cap, chunk) > 65535) chunk = ceil_div(ceil_div(Nc_cap, 65535), TILE) * TILE;
    size_t smem = static_cast<size_t>(KS) * STAGE_BYTES + 16 * QG * HG * 128 + 1024 + (hist ? 2048 * 4 : 0);
    // a CTA that takes all 512 TMEM columns must be alone on its SM: ask for
    // more than half of the SM's shared memory
    if (16 * QG * HG * NBD >= 512 && smem < 120 * 1024) smem = 120 * 1024;
    auto kern = index_tc_kernel<QG, NBD, KS, EG, HG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    const dim3 grid(static_cast<unsigned>(groups), static_cast<unsigned>(ceil_div(Nc_cap, chunk)));
    kern<<<grid, 64 + 128 * EG, smem, st>>>(tm_codes, tm_scales, q_codes, q_sf, w, q_pos, Tq, Nc_cap, m, chunk, scores,
                                            hist, hist_stride, bf16);
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

}  // namespace itc

}  // namespace

int index_take_device_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, itc::g_index_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        const int z = 0;
        cudaMemcpyToSymbol(itc::g_index_device_error, &z, sizeof(int));
    }
    return v;
}

namespace {
}  // namespace

// Decode index scores plus each row's key histogram (see index_tc_kernel); only
// the tensor-map path (c = 128, Hi = 4, Tq = 1) supports it.  HCA_ERR_UNSUPPORTED:
// nothing was launched.
int index_launch_hist(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                      const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                      int B, int64_t Nc_cap, int Hi, int c, int m, void* scores, uint32_t* hist,
                      int64_t hist_stride, cudaStream_t st, bool bf16) {
    if (c != 128 || (Hi != 4 && Hi != 64) || B <= 0 || Nc_cap <= 0) return HCA_ERR_UNSUPPORTED;
    float* sc = static_cast<float*>(scores);
    const int budget = launch_budget(HCA_BUDGET_DECODE_INDEX);
    if (Hi == 64)      // 16 head groups: N = 256 columns per buffer, two buffers fill TMEM (one CTA per SM)
        return itc::launch_tc<1, 2, 5, 2, 16>(q_codes, q_sf, w, k_codes, k_sf, q_pos, B, B, 1, Nc_cap, m, sc, st,
                                              budget > 0 ? std::min<int64_t>(budget, sm_count()) : sm_count(),
                                              hist, hist_stride, bf16 ? 1 : 0);
    return itc::launch_tc<1, 8, 5, 2>(q_codes, q_sf, w, k_codes, k_sf, q_pos, B, B, 1, Nc_cap, m, sc, st,
                                      budget > 0 ? budget : 2LL * sm_count(), hist, hist_stride, bf16 ? 1 : 0);
}

int index_launch(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                 const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                 int B, int Tq, int64_t Nc_cap, int Hi, int c, int m, void* scores_v,
                 cudaStream_t st, bool bf16) {
    if (B == 0 || Tq == 0 || Nc_cap == 0) return HCA_OK;
    float* scores = static_cast<float*>(scores_v);
    const int64_t rows = static_cast<int64_t>(B) * Tq;
    if (c == 128 && Hi == 64) {
        // the note's 64 indexer heads: one query per CTA, 16 head groups on the tensor pipe
        const int rc = itc::launch_tc<1, 2, 5, 2, 16>(q_codes, q_sf, w, k_codes, k_sf, q_pos, rows, B, Tq, Nc_cap, m,
                                                      scores, st, sm_count(), nullptr, 0, bf16 ? 1 : 0);
        return rc;   // (unaligned key buffers: HCA_ERR_UNSUPPORTED)
    }
    if (bf16 && !(c == 128 && Hi == 4)) return HCA_ERR_UNSUPPORTED;
    // enough blocks to fill the machine several times over for one row, but
    // a chunk of at least one warp step per warp
    int64_t chunk = 4096;
    const int64_t want_blocks = 4LL * sm_count();
    if (rows * ceil_div(Nc_cap, chunk) < want_blocks) {
        chunk = ceil_div(Nc_cap * rows, want_blocks);
        chunk = ceil_div(chunk, 128) * 128;
        if (chunk < 128) chunk = 128;
    }
    if (ceil_div(Nc_cap, chunk) > 65535) chunk = ceil_div(Nc_cap, 65535);
    const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(ceil_div(Nc_cap, chunk)));
    if (rows > 0x7FFFFFFFLL) return HCA_ERR_UNSUPPORTED;
    const bool small = Hi <= 4;
    if (c == 128 && Hi == 4) {
        // tensor cores on FP4 fed by the tensor memory accelerator: 16 queries per
        // CTA when a sequence has many query rows (prefill), else one.  Prefill: 16
        // epilogue warps (4 queries each per tile); with 8 the chunk's indexer took
        // 2.2 ms instead of 1.6 ms at prefill_4096_131k (the epilogue is latency bound)
        int rc;
        if (Tq % 16 == 0 && Tq >= 64)
            rc = itc::launch_tc<16, 2, 4, 4>(q_codes, q_sf, w, k_codes, k_sf, q_pos, rows, B, Tq, Nc_cap, m, scores, st,
                                             2LL * sm_count(), nullptr, 0, bf16 ? 1 : 0);
        else
            rc = itc::launch_tc<1, 8, 5, 2>(q_codes, q_sf, w, k_codes, k_sf, q_pos, rows, B, Tq, Nc_cap, m, scores, st,
                                            2LL * sm_count(), nullptr, 0, bf16 ? 1 : 0);
        if (rc != HCA_ERR_UNSUPPORTED || bf16) return rc;
        // unaligned key buffers: CUDA-core tensor path below
    }
    if (c == 128 && Hi == 4) {
        int64_t ch = 8192;
        if (rows * ceil_div(Nc_cap, ch) < want_blocks) {
            ch = ceil_div(Nc_cap * rows, want_blocks);
            ch = ceil_div(ch, 256) * 256;
            if (ch < 256) ch = 256;
        }
        if (ceil_div(Nc_cap, ch) > 65535) ch = ceil_div(ceil_div(Nc_cap, 65535), 16) * 16;
        const dim3 g2(static_cast<unsigned>(rows), static_cast<unsigned>(ceil_div(Nc_cap, ch)));
        index_mma_kernel<<<g2, kMmaWarps * 32, 0, st>>>(q_codes, q_sf, w, k_codes, k_sf, q_pos, Tq, Nc_cap, m, ch, scores);
    } else if (c == 128 && small)
        index_kernel<128, 4><<<grid, kWarps * 32, 0, st>>>(q_codes, q_sf, w, k_codes, k_sf, q_pos, Tq, Nc_cap, Hi, m, chunk, scores);
    else if (c == 128)
        index_kernel<128, 8><<<grid, kWarps * 32, 0, st>>>(q_codes, q_sf, w, k_codes, k_sf, q_pos, Tq, Nc_cap, Hi, m, chunk, scores);
    else if (c == 64 && small)
        index_kernel<64, 4><<<grid, kWarps * 32, 0, st>>>(q_codes, q_sf, w, k_codes, k_sf, q_pos, Tq, Nc_cap, Hi, m, chunk, scores);
    else if (c == 64)
        index_kernel<64, 8><<<grid, kWarps * 32, 0, st>>>(q_codes, q_sf, w, k_codes, k_sf, q_pos, Tq, Nc_cap, Hi, m, chunk, scores);
    else
        return HCA_ERR_UNSUPPORTED;
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

}  // namespace hca
