// compress.cu -- softmax-gated pooling of m raw tokens into one KV entry and
// its FP8/BF16 storage.
//
// "DeepSeek V4: Towards Highly Efficient Million Token Context Intelligence"
// (papers.chlience.com reading note), section 8 (HCA) compression equations
// S = Softmax_row(Z_block + B), C^Comp_i = sum_j S_j (.) C_j, section 7 (CSA,
// m = 4) and section 9 (RoPE dims BF16, the rest FP8).
//
// One thread owns 8 consecutive channels of one entry, so a 16-byte load
// brings 8 bf16 values of a token row and the D/8 threads of an entry read a
// token row fully coalesced.  The per-channel softmax is evaluated in the
// fixed fp32 sequence of the C ABI (include/hca.h) so the FP8 codes and
// scales are bit-exact: explicit __f*_rn intrinsics keep the compiler from
// contracting products into FMAs.
#include "common.cuh"

namespace hca {
namespace {

// E(z) ~= e^z for z <= 0: Cody & Waite argument reduction with a two-part
// ln 2, the Taylor series of e^r to degree 7 (Horner, fused multiply-adds),
// then the exact scale 2^n.  Constants: RN(1/ln 2); ln 2 rounded to fp32
// with its 9 low mantissa bits cleared (so n*LN2_HI is exact for |n| < 2^7);
// RN(ln 2 - LN2_HI); RN(1/k!) for k = 0..7.
__device__ __forceinline__ float cw_exp_neg(float z) {
    if (!(z >= -87.0f)) return 0.0f;
    const float kL2E = __uint_as_float(0x3FB8AA3Bu);
    const float kLn2Hi = __uint_as_float(0x3F317200u);
    const float kLn2Lo = __uint_as_float(0x35BFBE8Eu);
    float nf = rintf(__fmul_rn(z, kL2E));
    float r = __fmaf_rn(-nf, kLn2Hi, z);
    r = __fmaf_rn(-nf, kLn2Lo, r);
    float p = __uint_as_float(0x39500D01u);                 // 1/7!
    p = __fmaf_rn(p, r, __uint_as_float(0x3AB60B61u));      // 1/6!
    p = __fmaf_rn(p, r, __uint_as_float(0x3C088889u));      // 1/5!
    p = __fmaf_rn(p, r, __uint_as_float(0x3D2AAAABu));      // 1/4!
    p = __fmaf_rn(p, r, __uint_as_float(0x3E2AAAABu));      // 1/3!
    p = __fmaf_rn(p, r, 0.5f);                              // 1/2!
    p = __fmaf_rn(p, r, 1.0f);                              // 1/1!
    p = __fmaf_rn(p, r, 1.0f);                              // 1/0!
    const int n = static_cast<int>(nf);                     // -126 <= n <= 0
    return __fmul_rn(p, __uint_as_float(static_cast<uint32_t>(n + 127) << 23));
}

__device__ __forceinline__ void load8_bf16(const uint16_t* p, float (&v)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void load8_f32(const float* p, float (&v)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int kThreads = 256;

// M tokens per block, D channels per entry.  Requires D % 8 == 0,
// (D - d_rope) % g == 0, g % 8 == 0, g <= 256 (a group lives in one warp).
template <int M, int D>
__global__ void __launch_bounds__(kThreads)
pool_quant_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ gate,
                  int64_t seq_stride, const float* __restrict__ bias,
                  int64_t n_entries_total, int64_t n_blocks, int d_rope, int g,
                  uint8_t* __restrict__ codes, float* __restrict__ scales,
                  uint16_t* __restrict__ rope, int64_t cap, int64_t entry_begin) {
    constexpr int TPE = D / 8;              // threads per entry
    constexpr int EPB = kThreads / TPE;     // entries per block
    const int ch = (threadIdx.x % TPE) * 8; // first channel of this thread
    int64_t e = static_cast<int64_t>(blockIdx.x) * EPB + threadIdx.x / TPE;
    const bool valid = e < n_entries_total;
    if (!valid) e = 0;                      // compute on entry 0, store nothing
    const int64_t b = e / n_blocks, j = e % n_blocks;
    const size_t row0 = (static_cast<size_t>(b) * seq_stride + static_cast<size_t>(j) * M) * D + ch;
    const uint16_t* xp = x + row0;
    const uint16_t* gp = gate + row0;
    const float* bp = bias + ch;

    float zmax[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) zmax[c] = -INFINITY;
    constexpr bool kCacheZ = M <= 8;
    float zc[kCacheZ ? M : 1][8];
#pragma unroll(kCacheZ ? M : 4)
    for (int i = 0; i < M; ++i) {
        float gv[8], bv[8];
        load8_bf16(gp + static_cast<size_t>(i) * D, gv);
        load8_f32(bp + static_cast<size_t>(i) * D, bv);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float z = __fadd_rn(gv[c], bv[c]);
            if (kCacheZ) zc[kCacheZ ? i : 0][c] = z;
            zmax[c] = fmaxf(zmax[c], z);
        }
    }
    float S[8], N[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) { S[c] = 0.0f; N[c] = 0.0f; }
#pragma unroll(kCacheZ ? M : 4)
    for (int i = 0; i < M; ++i) {
        float xv[8], z[8];
        load8_bf16(xp + static_cast<size_t>(i) * D, xv);
        if (kCacheZ) {
#pragma unroll
            for (int c = 0; c < 8; ++c) z[c] = zc[kCacheZ ? i : 0][c];
        } else {
            float gv[8], bv[8];
            load8_bf16(gp + static_cast<size_t>(i) * D, gv);
            load8_f32(bp + static_cast<size_t>(i) * D, bv);
#pragma unroll
            for (int c = 0; c < 8; ++c) z[c] = __fadd_rn(gv[c], bv[c]);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float ev = cw_exp_neg(__fsub_rn(z[c], zmax[c]));
            S[c] = __fadd_rn(S[c], ev);
            N[c] = __fadd_rn(N[c], __fmul_rn(ev, xv[c]));
        }
    }
    float y[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) y[c] = __fdiv_rn(N[c], S[c]);

    // ---- storage: FP8 groups of g channels, bf16 RoPE tail
    const int dn = D - d_rope;
    const int tpg = g / 8;                  // threads per scale group
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) amax = fmaxf(amax, fabsf(y[c]));
    for (int o = 1; o < tpg; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));

    const size_t erow = static_cast<size_t>(b) * cap + static_cast<size_t>(entry_begin + j);
    if (!valid) return;
    if (ch < dn) {
        const float scale = __fdiv_rn(amax, 448.0f);
        uint32_t w0 = 0, w1 = 0;
        if (amax != 0.0f) {
            uint16_t p0 = f32x2_to_e4m3x2(__fdiv_rn(y[0], scale), __fdiv_rn(y[1], scale));
            uint16_t p1 = f32x2_to_e4m3x2(__fdiv_rn(y[2], scale), __fdiv_rn(y[3], scale));
            uint16_t p2 = f32x2_to_e4m3x2(__fdiv_rn(y[4], scale), __fdiv_rn(y[5], scale));
            uint16_t p3 = f32x2_to_e4m3x2(__fdiv_rn(y[6], scale), __fdiv_rn(y[7], scale));
            w0 = static_cast<uint32_t>(p0) | (static_cast<uint32_t>(p1) << 16);
            w1 = static_cast<uint32_t>(p2) | (static_cast<uint32_t>(p3) << 16);
        }
        *reinterpret_cast<uint2*>(codes + erow * dn + ch) = make_uint2(w0, w1);
        if ((ch % g) == 0) scales[erow * (dn / g) + ch / g] = scale;
    } else {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(rope + erow * d_rope + (ch - dn)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <int M, int D>
int launch_pool(const uint16_t* x, const uint16_t* gate, int64_t seq_stride, const float* bias,
                int B, int64_t n_blocks, int d_rope, int g, const hca_kv_cache& out,
                int64_t entry_begin, cudaStream_t st) {
    const int64_t total = static_cast<int64_t>(B) * n_blocks;
    if (total == 0) return HCA_OK;
    constexpr int EPB = kThreads / (D / 8);
    const int64_t grid = ceil_div(total, EPB);
    pool_quant_kernel<M, D><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(
        x, gate, seq_stride, bias, total, n_blocks, d_rope, g, out.codes, out.scales, out.rope,
        out.capacity, entry_begin);
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

}  // namespace

int compress_launch(int m, const uint16_t* x, const uint16_t* gate, int64_t seq_stride,
                    const float* bias, int B, int64_t n_blocks, const hca_kv_layout& L,
                    const hca_kv_cache& out, int64_t entry_begin, cudaStream_t st) {
    if (L.d == 512) {
        if (m == 4) return launch_pool<4, 512>(x, gate, seq_stride, bias, B, n_blocks, L.d_rope, L.scale_group, out, entry_begin, st);
        if (m == 128) return launch_pool<128, 512>(x, gate, seq_stride, bias, B, n_blocks, L.d_rope, L.scale_group, out, entry_begin, st);
    } else if (L.d == 128) {
        if (m == 4) return launch_pool<4, 128>(x, gate, seq_stride, bias, B, n_blocks, L.d_rope, L.scale_group, out, entry_begin, st);
        if (m == 128) return launch_pool<128, 128>(x, gate, seq_stride, bias, B, n_blocks, L.d_rope, L.scale_group, out, entry_begin, st);
    }
    return HCA_ERR_UNSUPPORTED;
}

}  // namespace hca
