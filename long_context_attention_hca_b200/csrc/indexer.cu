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

// 2^(e) for an integer exponent, exact; e outside the normal range goes through ldexpf.
__device__ __forceinline__ float pow2i(int e) {
    if (e >= -126 && e <= 127) return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
    return ldexpf(1.0f, e);
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
                const float t = __fmul_rn(static_cast<float>(acc), pow2i(qe[h] + ke[j] - 2));
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
                tA[j][r] = __fmul_rn(D0[j + 2 * r], pow2i(eqv[0][j] + ekA));
                tB[j][r] = __fmul_rn(D1[j + 2 * r], pow2i(eqv[1][j] + ekB));
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

}  // namespace

int index_launch(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                 const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                 int B, int Tq, int64_t Nc_cap, int Hi, int c, int m, float* scores,
                 cudaStream_t st) {
    if (B == 0 || Tq == 0 || Nc_cap == 0) return HCA_OK;
    const int64_t rows = static_cast<int64_t>(B) * Tq;
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
