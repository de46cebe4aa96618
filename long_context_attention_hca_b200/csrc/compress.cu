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

// Section 9 extras of one stored vector (a pooled entry or a window token),
// applied to the 8 channels y[] this thread owns (channels ch .. ch+7; the
// TPE threads of the vector are consecutive lanes, two warps for D = 512).
//  - RMSNorm (norm_w != null) in the fixed fp32 sequence of the C ABI: the
//    squares are rounded, summed as a pairwise tree over consecutive pairs
//    (inside the thread, then a butterfly over its lanes, then the two warps
//    of a D = 512 vector through shared memory), r = sqrt(ss / D + eps)
//    correctly rounded, y = (y / r) * w.  Every thread of the block must call
//    it (warp shuffles and a block barrier).
template <int D>
__device__ __forceinline__ void rms_norm8(float (&y)[8], const float* __restrict__ norm_w, float eps, int ch,
                                          float* s_part) {
    constexpr int TPE = D / 8;
    float sq[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) sq[c] = __fmul_rn(y[c], y[c]);
    float s = __fadd_rn(__fadd_rn(__fadd_rn(sq[0], sq[1]), __fadd_rn(sq[2], sq[3])),
                        __fadd_rn(__fadd_rn(sq[4], sq[5]), __fadd_rn(sq[6], sq[7])));
#pragma unroll
    for (int o = 1; o < (TPE < 32 ? TPE : 32); o <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
    if (TPE > 32) {
        // lanes of warp 2v hold channels [0, 256) of vector v, warp 2v+1 [256, 512)
        const int wv = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) s_part[wv] = s;
        __syncthreads();
        s = __fadd_rn(s_part[wv & ~1], s_part[wv | 1]);
        __syncthreads();
    }
    const float r = __fsqrt_rn(__fadd_rn(__fdiv_rn(s, static_cast<float>(D)), eps));
    float w[8];
    load8_f32(norm_w + ch, w);
#pragma unroll
    for (int c = 0; c < 8; ++c) y[c] = __fmul_rn(__fdiv_rn(y[c], r), w[c]);
}

//  - Partial RoPE of the thread's 4 channel pairs (2i, 2i+1) of the RoPE
//    dims, rotated to position pos by the angle pos * inv_freq[i] (an exact
//    fp64 product), in fp64 with every product and sum rounded (no FMA), then
//    rounded once to bf16 (4 bf16x2 words out).
__device__ __forceinline__ void rope8_to_bf16(const float (&y)[8], int pair0, int64_t pos,
                                              const float* __restrict__ inv_freq, uint32_t (&out)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const double ang = __dmul_rn(static_cast<double>(pos), static_cast<double>(__ldg(inv_freq + pair0 + i)));
        double sn, cs;
        sincos(ang, &sn, &cs);
        const double a = y[2 * i], b = y[2 * i + 1];
        const double x0 = __dsub_rn(__dmul_rn(a, cs), __dmul_rn(b, sn));
        const double x1 = __dadd_rn(__dmul_rn(a, sn), __dmul_rn(b, cs));
        const uint32_t lo = __bfloat16_as_ushort(__double2bfloat16(x0));
        const uint32_t hi = __bfloat16_as_ushort(__double2bfloat16(x1));
        out[i] = lo | (hi << 16);
    }
}

// M tokens per block, D channels per entry.  Requires D % 8 == 0,
// (D - d_rope) % g == 0, g % 8 == 0, g <= 256 (a group lives in one warp).
template <int M, int D>
__global__ void __launch_bounds__(kThreads)
pool_quant_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ gate,
                  int64_t seq_stride, const float* __restrict__ bias,
                  int64_t n_entries_total, int64_t n_blocks, int d_rope, int g,
                  uint8_t* __restrict__ codes, float* __restrict__ scales,
                  uint16_t* __restrict__ rope, int64_t cap, int64_t entry_begin,
                  const float* __restrict__ norm_w, float norm_eps, const float* __restrict__ inv_freq) {
    __shared__ float s_part[kThreads / 32];
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
    if (norm_w) rms_norm8<D>(y, norm_w, norm_eps, ch, s_part);     // uniform over the grid

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
        if (inv_freq) {
            // the entry's position: its block's first token
            rope8_to_bf16(y, (ch - dn) / 2, (entry_begin + j) * M, inv_freq, w);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
                w[i] = *reinterpret_cast<uint32_t*>(&h);
            }
        }
        *reinterpret_cast<uint4*>(rope + erow * d_rope + (ch - dn)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// One window token per TPE threads: RMSNorm and partial RoPE at the token's
// position (the same sequences as a stored entry), all channels out as bf16.
template <int D>
__global__ void __launch_bounds__(kThreads)
token_prep_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ pos, int64_t n, int d_rope,
                  const float* __restrict__ norm_w, float norm_eps, const float* __restrict__ inv_freq,
                  uint16_t* __restrict__ out) {
    __shared__ float s_part[kThreads / 32];
    constexpr int TPE = D / 8;
    constexpr int EPB = kThreads / TPE;
    const int ch = (threadIdx.x % TPE) * 8;
    int64_t t = static_cast<int64_t>(blockIdx.x) * EPB + threadIdx.x / TPE;
    const bool valid = t < n;
    if (!valid) t = 0;
    float y[8];
    load8_bf16(x + static_cast<size_t>(t) * D + ch, y);
    if (norm_w) rms_norm8<D>(y, norm_w, norm_eps, ch, s_part);
    if (!valid) return;
    const int dn = D - d_rope;
    uint32_t w[4];
    if (ch >= dn && inv_freq) {
        rope8_to_bf16(y, (ch - dn) / 2, pos[t], inv_freq, w);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
    }
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * D + ch) = make_uint4(w[0], w[1], w[2], w[3]);
}

template <int M, int D>
int launch_pool(const uint16_t* x, const uint16_t* gate, int64_t seq_stride, const float* bias,
                int B, int64_t n_blocks, int d_rope, int g, const hca_kv_cache& out,
                int64_t entry_begin, const hca_entry_extras* ex, cudaStream_t st) {
    const int64_t total = static_cast<int64_t>(B) * n_blocks;
    if (total == 0) return HCA_OK;
    constexpr int EPB = kThreads / (D / 8);
    const int64_t grid = ceil_div(total, EPB);
    pool_quant_kernel<M, D><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(
        x, gate, seq_stride, bias, total, n_blocks, d_rope, g, out.codes, out.scales, out.rope,
        out.capacity, entry_begin, ex ? ex->norm_w : nullptr, ex ? ex->norm_eps : 0.0f,
        ex ? ex->inv_freq : nullptr);
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

}  // namespace

int compress_launch(int m, const uint16_t* x, const uint16_t* gate, int64_t seq_stride,
                    const float* bias, int B, int64_t n_blocks, const hca_kv_layout& L,
                    const hca_kv_cache& out, int64_t entry_begin, const hca_entry_extras* ex, cudaStream_t st) {
    if (L.d == 512) {
        if (m == 4) return launch_pool<4, 512>(x, gate, seq_stride, bias, B, n_blocks, L.d_rope, L.scale_group, out, entry_begin, ex, st);
        if (m == 128) return launch_pool<128, 512>(x, gate, seq_stride, bias, B, n_blocks, L.d_rope, L.scale_group, out, entry_begin, ex, st);
    } else if (L.d == 128) {
        if (m == 4) return launch_pool<4, 128>(x, gate, seq_stride, bias, B, n_blocks, L.d_rope, L.scale_group, out, entry_begin, ex, st);
        if (m == 128) return launch_pool<128, 128>(x, gate, seq_stride, bias, B, n_blocks, L.d_rope, L.scale_group, out, entry_begin, ex, st);
    }
    return HCA_ERR_UNSUPPORTED;
}

namespace {

// ---------------------------------------------------------------- overlapped compressor
// "DeepSeek V4 ..." note, section 7: CSA's two KV streams C_a, C_b and gate
// streams Z_a, Z_b; each entry pools 2m adjacent tokens with one softmax.
// Entry entry_begin + j pools the m tokens of block j-1 from stream a (rows
// (j-1)m .. jm-1 of xa/za, or rows 0..m-1 of a_prev/za_prev for j = 0, absent
// when a_prev is null) and the m tokens of block j from stream b (rows jm ..
// jm+m-1 of xb/zb), with bias rows 0..m-1 for the a-half and m..2m-1 for the
// b-half, in the fp32 sequence of pool_quant_kernel over the 2m tokens in
// that order.  OUT_KEY: the pooled c-vector is an indexer key, stored FP4
// (OCP MX e2m1 with one ue8m0 exponent per 32 elements, X = floor(log2
// amax) - 2, codes e2m1(v / 2^X) nearest-even saturating at 6); otherwise an
// entry stored FP8/BF16 as pool_quant_kernel stores it.
template <int M, int D, bool OUT_KEY>
__global__ void __launch_bounds__(kThreads)
pool_overlap_kernel(const uint16_t* __restrict__ xa, const uint16_t* __restrict__ za,
                    const uint16_t* __restrict__ xb, const uint16_t* __restrict__ zb,
                    const uint16_t* __restrict__ a_prev, const uint16_t* __restrict__ za_prev,
                    int64_t seq_stride, const float* __restrict__ bias, int64_t n_entries_total, int64_t n_blocks,
                    int d_rope, int g, uint8_t* __restrict__ codes, float* __restrict__ scales,
                    uint16_t* __restrict__ rope, uint8_t* __restrict__ k_sf, int64_t cap, int64_t entry_begin) {
    constexpr int TPE = D / 8;
    constexpr int EPB = kThreads / TPE;
    const int ch = (threadIdx.x % TPE) * 8;
    int64_t e = static_cast<int64_t>(blockIdx.x) * EPB + threadIdx.x / TPE;
    const bool valid = e < n_entries_total;
    if (!valid) e = 0;
    const int64_t b = e / n_blocks, j = e % n_blocks;
    const size_t seq = static_cast<size_t>(b) * seq_stride;
    const uint16_t* ax = nullptr;
    const uint16_t* az = nullptr;
    if (j >= 1) {
        ax = xa + (seq + static_cast<size_t>(j - 1) * M) * D + ch;
        az = za + (seq + static_cast<size_t>(j - 1) * M) * D + ch;
    } else if (a_prev) {
        ax = a_prev + seq * D + ch;
        az = za_prev + seq * D + ch;
    }
    const uint16_t* bx = xb + (seq + static_cast<size_t>(j) * M) * D + ch;
    const uint16_t* bz = zb + (seq + static_cast<size_t>(j) * M) * D + ch;
    const bool has_a = ax != nullptr;
    float z[2 * M][8];
    float zmax[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) zmax[c] = -INFINITY;
#pragma unroll
    for (int i = 0; i < 2 * M; ++i) {
        const bool a_half = i < M;
        if (a_half && !has_a) continue;
        float gv[8], bv[8];
        load8_bf16(a_half ? az + static_cast<size_t>(i) * D : bz + static_cast<size_t>(i - M) * D, gv);
        load8_f32(bias + static_cast<size_t>(i) * D + ch, bv);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            z[i][c] = __fadd_rn(gv[c], bv[c]);
            zmax[c] = fmaxf(zmax[c], z[i][c]);
        }
    }
    float S[8], N[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) { S[c] = 0.0f; N[c] = 0.0f; }
#pragma unroll
    for (int i = 0; i < 2 * M; ++i) {
        const bool a_half = i < M;
        if (a_half && !has_a) continue;
        float xv[8];
        load8_bf16(a_half ? ax + static_cast<size_t>(i) * D : bx + static_cast<size_t>(i - M) * D, xv);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float ev = cw_exp_neg(__fsub_rn(z[i][c], zmax[c]));
            S[c] = __fadd_rn(S[c], ev);
            N[c] = __fadd_rn(N[c], __fmul_rn(ev, xv[c]));
        }
    }
    float y[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) y[c] = __fdiv_rn(N[c], S[c]);

    const size_t erow = static_cast<size_t>(b) * cap + static_cast<size_t>(entry_begin + j);
    if (OUT_KEY) {
        // FP4: 4 threads (32 channels) share one exponent
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < 8; ++c) amax = fmaxf(amax, fabsf(y[c]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        if (!valid) return;
        int X = -127;
        const uint32_t ebits = (__float_as_uint(amax) >> 23) & 0xFFu;
        if (amax > 0.0f && ebits > 0u) X = max(-127, static_cast<int>(ebits) - 127 - 2);
        const float inv = ldexpf(1.0f, -X);
        uint32_t word;
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
            "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
            : "=r"(word)
            : "f"(__fmul_rn(y[0], inv)), "f"(__fmul_rn(y[1], inv)), "f"(__fmul_rn(y[2], inv)),
              "f"(__fmul_rn(y[3], inv)), "f"(__fmul_rn(y[4], inv)), "f"(__fmul_rn(y[5], inv)),
              "f"(__fmul_rn(y[6], inv)), "f"(__fmul_rn(y[7], inv)));
        *reinterpret_cast<uint32_t*>(codes + erow * (D / 2) + ch / 2) = word;     // element 2i: low nibble
        if ((ch & 31) == 0) k_sf[erow * (D / 32) + ch / 32] = static_cast<uint8_t>(X + 127);
        return;
    }
    const int dn = D - d_rope;
    const int tpg = g / 8;
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) amax = fmaxf(amax, fabsf(y[c]));
    for (int o = 1; o < tpg; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
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

// one 16-byte vector (8 channels) per thread: the token into the window ring
// and the block tail
__global__ void state_append_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ gate,
                                    const uint16_t* __restrict__ win_x, int B, int d, int64_t pos,
                                    uint16_t* __restrict__ window, int W, uint16_t* __restrict__ tail_x,
                                    uint16_t* __restrict__ tail_gate, int m) {
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    const int per = d / 8;
    if (v >= B * per) return;
    const int b = v / per, c = (v % per) * 8;
    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(b) * d + c));
    const uint4 wv = win_x ? __ldg(reinterpret_cast<const uint4*>(win_x + static_cast<size_t>(b) * d + c)) : xv;
    if (W > 0)
        *reinterpret_cast<uint4*>(window + (static_cast<size_t>(b) * W + pos % W) * d + c) = wv;
    if (m > 0 && tail_x) {
        const size_t r = (static_cast<size_t>(b) * m + pos % m) * d + c;
        *reinterpret_cast<uint4*>(tail_x + r) = xv;
        *reinterpret_cast<uint4*>(tail_gate + r) =
            __ldg(reinterpret_cast<const uint4*>(gate + static_cast<size_t>(b) * d + c));
    }
}
}  // namespace

int overlap_launch(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                   const uint16_t* a_prev, const uint16_t* za_prev, int64_t seq_stride, const float* bias, int B,
                   int64_t n_blocks, int D, int d_rope, int g, uint8_t* codes, float* scales, uint16_t* rope,
                   uint8_t* k_sf, int64_t cap, int64_t entry_begin, bool key, cudaStream_t st) {
    const int64_t total = static_cast<int64_t>(B) * n_blocks;
    if (total == 0) return HCA_OK;
    const unsigned grid = static_cast<unsigned>(ceil_div(total, kThreads / (D / 8)));
#define HCA_OVL(DD, KEY)                                                                                     \
    pool_overlap_kernel<4, DD, KEY><<<grid, kThreads, 0, st>>>(xa, za, xb, zb, a_prev, za_prev, seq_stride, bias, \
                                                              total, n_blocks, d_rope, g, codes, scales, rope,  \
                                                              k_sf, cap, entry_begin)
    if (key) {
        if (D == 128) HCA_OVL(128, true);
        else if (D == 64) HCA_OVL(64, true);
        else return HCA_ERR_UNSUPPORTED;
    } else {
        if (D == 512) HCA_OVL(512, false);
        else if (D == 128) HCA_OVL(128, false);
        else return HCA_ERR_UNSUPPORTED;
    }
#undef HCA_OVL
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

int state_append_launch(const uint16_t* x, const uint16_t* gate, const uint16_t* win_x, int B, int d, int64_t pos,
                        uint16_t* window, int W, uint16_t* tail_x, uint16_t* tail_gate, int m, cudaStream_t st) {
    const int n = B * (d / 8);
    if (n == 0) return HCA_OK;
    state_append_kernel<<<(n + 255) / 256, 256, 0, st>>>(x, gate, win_x, B, d, pos, window, W, tail_x, tail_gate, m);
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

int token_prep_launch(const uint16_t* x, const int32_t* pos, int64_t n, const hca_kv_layout& L,
                      const hca_entry_extras* ex, uint16_t* out, cudaStream_t st) {
    if (n == 0) return HCA_OK;
    const float* nw = ex ? ex->norm_w : nullptr;
    const float* fq = ex ? ex->inv_freq : nullptr;
    const float eps = ex ? ex->norm_eps : 0.0f;
    if (L.d == 512) {
        token_prep_kernel<512><<<static_cast<unsigned>(ceil_div(n, kThreads / 64)), kThreads, 0, st>>>(
            x, pos, n, L.d_rope, nw, eps, fq, out);
    } else if (L.d == 128) {
        token_prep_kernel<128><<<static_cast<unsigned>(ceil_div(n, kThreads / 16)), kThreads, 0, st>>>(
            x, pos, n, L.d_rope, nw, eps, fq, out);
    } else {
        return HCA_ERR_UNSUPPORTED;
    }
    HCA_CHECK_LAUNCH();
    return HCA_OK;
}

}  // namespace hca
