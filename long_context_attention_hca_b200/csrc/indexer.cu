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
constexpr int kMaxHi = 8;

template <int C>
__global__ void __launch_bounds__(kWarps * 32)
index_kernel(const uint8_t* __restrict__ q_codes, const uint8_t* __restrict__ q_sf,
             const float* __restrict__ w, const uint8_t* __restrict__ k_codes,
             const uint8_t* __restrict__ k_sf, const int32_t* __restrict__ q_pos,
             int Tq, int64_t Nc_cap, int Hi, int m, int64_t chunk, float* __restrict__ scores) {
    constexpr int NB = C / 32;               // blocks per entry = lanes per entry
    constexpr int EPW = 32 / NB;             // entries per warp step
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int blk = lane % NB;
    const int64_t qrow = blockIdx.x;         // b * Tq + t (rows on x: neighbours share a key chunk in L2)
    const int64_t b = qrow / Tq;

    // query expansion for this lane's block, all heads
    uint32_t qv[kMaxHi][8];
    int qe[kMaxHi];
    float wh[kMaxHi];
#pragma unroll
    for (int h = 0; h < kMaxHi; ++h) {
        if (h < Hi) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(q_codes + ((qrow * Hi + h) * C / 2) + blk * 16));
            fp4x8_to_i8x8(u.x, qv[h][0], qv[h][1]);
            fp4x8_to_i8x8(u.y, qv[h][2], qv[h][3]);
            fp4x8_to_i8x8(u.z, qv[h][4], qv[h][5]);
            fp4x8_to_i8x8(u.w, qv[h][6], qv[h][7]);
            qe[h] = static_cast<int>(__ldg(q_sf + (qrow * Hi + h) * NB + blk));
            wh[h] = __ldg(w + qrow * Hi + h);
        }
    }
    const int64_t pos = q_pos[qrow];
    int64_t elig = (pos + 1) / m;
    elig = elig < 0 ? 0 : (elig > Nc_cap ? Nc_cap : elig);

    const int64_t s_begin = static_cast<int64_t>(blockIdx.y) * chunk;
    const int64_t s_end = min(s_begin + chunk, Nc_cap);
    const uint8_t* kc_base = k_codes + static_cast<size_t>(b) * Nc_cap * (C / 2);
    const uint8_t* ks_base = k_sf + static_cast<size_t>(b) * Nc_cap * NB;
    float* out = scores + static_cast<size_t>(qrow) * Nc_cap;

    for (int64_t s0 = s_begin + warp * EPW; s0 < s_end; s0 += kWarps * EPW) {
        const int64_t s = s0 + lane / NB;
        const bool live = s < s_end && s < elig;
        float t[kMaxHi];
        if (live) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(kc_base + s * (C / 2) + blk * 16));
            uint32_t kv[8];
            fp4x8_to_i8x8(u.x, kv[0], kv[1]);
            fp4x8_to_i8x8(u.y, kv[2], kv[3]);
            fp4x8_to_i8x8(u.z, kv[4], kv[5]);
            fp4x8_to_i8x8(u.w, kv[6], kv[7]);
            const int ke = static_cast<int>(__ldg(ks_base + s * NB + blk));
#pragma unroll
            for (int h = 0; h < kMaxHi; ++h) {
                if (h < Hi) {
                    int acc = 0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc = __dp4a(static_cast<int>(kv[i]), static_cast<int>(qv[h][i]), acc);
                    // block dot = acc / 4 exactly; times 2^(eq + ek - 254)
                    t[h] = __fmul_rn(static_cast<float>(acc), pow2i(qe[h] + ke - 254 - 2));
                }
            }
        } else {
#pragma unroll
            for (int h = 0; h < kMaxHi; ++h) t[h] = 0.0f;
        }
        // ordered block sum on the entry's first lane: ((t0 + t1) + t2) + t3
        float dot[kMaxHi];
#pragma unroll
        for (int h = 0; h < kMaxHi; ++h) {
            if (h < Hi) {
                float acc = t[h];
#pragma unroll
                for (int j = 1; j < NB; ++j) acc = __fadd_rn(acc, __shfl_down_sync(0xffffffffu, t[h], j));
                dot[h] = acc;
            }
        }
        if (blk == 0 && s < s_end) {
            float sc;
            if (s < elig) {
                sc = 0.0f;
#pragma unroll
                for (int h = 0; h < kMaxHi; ++h) {
                    if (h < Hi) {
                        const float r = dot[h] > 0.0f ? dot[h] : 0.0f;
                        sc = __fadd_rn(sc, __fmul_rn(wh[h], r));
                    }
                }
            } else {
                sc = -INFINITY;
            }
            out[s] = sc;
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
    int64_t chunk = 2048;
    const int64_t want_blocks = 4LL * sm_count();
    if (rows * ceil_div(Nc_cap, chunk) < want_blocks) {
        chunk = ceil_div(Nc_cap * rows, want_blocks);
        chunk = ceil_div(chunk, 128) * 128;
        if (chunk < 128) chunk = 128;
    }
    if (ceil_div(Nc_cap, chunk) > 65535) chunk = ceil_div(Nc_cap, 65535);
    const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(ceil_div(Nc_cap, chunk)));
    if (rows > 0x7FFFFFFFLL) return HCA_ERR_UNSUPPORTED;
    if (c == 128)
        index_kernel<128><<<grid, kWarps * 32, 0, st>>>(q_codes, q_sf, w, k_codes, k_sf, q_pos, Tq, Nc_cap, Hi, m, chunk, scores);
    else if (c == 64)
        index_kernel<64><<<grid, kWarps * 32, 0, st>>>(q_codes, q_sf, w, k_codes, k_sf, q_pos, Tq, Nc_cap, Hi, m, chunk, scores);
    else
        return HCA_ERR_UNSUPPORTED;
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

}  // namespace hca
