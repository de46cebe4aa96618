// attention.cu -- core attention of CSA and HCA over compressed entries plus
// the sliding window, for decode (split-K + log-sum-exp combine) and
// chunked prefill.
//
// "DeepSeek V4: Towards Highly Efficient Million Token Context Intelligence"
// (papers.chlience.com reading note), section 7: shared key-value MQA (the
// compressed entry is both key and value), the sliding-window branch over the
// last n_win uncompressed tokens; section 8: HCA attends densely to every
// compressed entry; section 9: entries stored FP8 (codes x fp32 scale) with
// BF16 RoPE dims.  One joint softmax covers compressed keys and window keys.
//
// This file holds the portable tensor-core path (mma.sync m16n8k16, fp16
// operands, fp32 accumulation).  A work unit is one query token with its H
// heads (decode: one sequence; prefill: one position) and a list of key
// "slots": the unit's compressed keys first, then its window tokens.  A CTA
// takes one (unit, split) pair, stages 64-key tiles in shared memory
// (dequantised to fp16), and keeps the online-softmax state and the fp32
// output accumulator in registers:  warp (hg, half) owns heads
// 16*hg .. 16*hg+15 and output dims half*D/2 .. ; the two halves exchange
// their partial q.k sums through shared memory so both see the same logits.
#include <mutex>

#include "common.cuh"

namespace hca {
namespace attn {

constexpr int TK = 64;  // keys per tile

struct Params {
    const uint16_t* q;          // [units][H][D] bf16
    int H;
    const uint8_t* codes;       // cache SoA
    const float* scales;
    const uint16_t* rope;
    int64_t cap;                // entries per sequence
    int d_rope, g;
    int prefill;                // 0: decode (unit = sequence), 1: prefill (unit = position)
    const int32_t* idx;         // sparse keys [units][idx_stride] or null (dense)
    int idx_stride;
    const int32_t* n_comp;      // decode: [units]; prefill sparse: count [units]
    int dense_m;                // prefill dense: eligible = min(cap, (p+1)/m)
    int p0;                     // prefill: position of unit 0
    const uint16_t* win;        // decode: [units][W][D]; prefill: raw [(W-1)+units][D]
    int W;
    float scale_log2;           // softmax_scale * log2(e)
    int n_splits, tiles_per_split;
    uint16_t* out;              // [units][H][D]
    float* lse;                 // [units][H] or null
    float* part_o;              // [units][splits][HP][D]
    float* part_ml;             // [units][splits][2][HP]
    // section 9 extras (each null when off)
    const float* q_norm_w;      // [D] query-head RMSNorm weight
    float norm_eps;
    const float* sink;          // [H] sink logit per head (natural log)
    const float* inv_freq;      // [d_rope/2] RoPE frequencies
    const int32_t* q_pos;       // decode: [units] query positions
    const int32_t* win_len;     // decode: [units] valid window rows (<= W), or null: W
};

constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ int64_t unit_pos(const Params& p, int64_t u) {
    return p.prefill ? static_cast<int64_t>(p.p0) + u : (p.q_pos ? static_cast<int64_t>(p.q_pos[u]) : 0);
}

__device__ __forceinline__ void rope_cs(const float* inv_freq, int i, int64_t t, float& c, float& s) {
    double sn, cs;
    sincos(static_cast<double>(t) * static_cast<double>(__ldg(inv_freq + i)), &sn, &cs);
    c = static_cast<float>(cs);
    s = static_cast<float>(sn);
}

template <int D, int HP>
struct Cfg {
    static constexpr int NHG = HP / 16;
    static constexpr int NWARPS = NHG * 2;
    static constexpr int NTHREADS = NWARPS * 32;
    static constexpr int DH = D / 2;            // output dims per warp
    static constexpr int NT_O = DH / 8;         // n-tiles of the output accumulator
    static constexpr int KS_QK = DH / 16;       // k-steps of the partial q.k
    static constexpr int CHUNKS = D / 8;        // 16-byte chunks per fp16 row
    static constexpr size_t Q_BYTES = size_t(HP) * D * 2;
    static constexpr size_t K_BYTES = size_t(TK) * D * 2;
    static constexpr size_t X_BYTES = size_t(NWARPS) * 32 * 32 * 4;
    static constexpr size_t SMEM = Q_BYTES + K_BYTES + X_BYTES;
};

// fp16 row-major tile with 16-byte chunks XOR-swizzled by row (conflict-free ldmatrix).
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return static_cast<uint32_t>(row * (D * 2) + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Per-unit key list: n_c compressed keys then n_w window tokens (rows of `wrow`).
struct UnitKeys {
    int n_c, n_w;
    const int32_t* ent;          // sparse list or null (dense: entry = slot)
    int64_t kv_row0;             // first cache row of the unit's sequence
    const uint16_t* wrow;        // first window row
};

__device__ __forceinline__ UnitKeys unit_keys(const Params& p, int64_t u, int D) {
    UnitKeys k;
    if (!p.prefill) {
        int nc = p.n_comp[u];
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
            int64_t e = (pos + 1) / p.dense_m;
            k.n_c = static_cast<int>(e > p.cap ? p.cap : e);
            k.ent = nullptr;
        }
        k.kv_row0 = 0;
        const int64_t first = pos - (p.W - 1) > 0 ? pos - (p.W - 1) : 0;
        // raw row r holds position p0 - (W-1) + r
        k.wrow = p.win + static_cast<size_t>(first - (p.p0 - (p.W - 1))) * D;
        k.n_w = static_cast<int>(pos - first + 1);
    }
    return k;
}

// Stage keys [slot0, slot0 + TK) of a unit into an fp16 swizzled tile.
template <int D, int NTHREADS>
__device__ __forceinline__ void load_tile(const Params& p, const UnitKeys& uk, int slot0, char* ks) {
    constexpr int C16 = D / 16;                 // 16-value groups per row
    const int dn = D - p.d_rope, ng = dn / p.g;
    for (int w = threadIdx.x; w < TK * C16; w += NTHREADS) {
        const int r = w / C16, c = w % C16;
        const int slot = slot0 + r;
        uint32_t h[8];
        if (slot < uk.n_c) {
            int64_t e = uk.ent ? uk.ent[slot] : slot;
            if (e < 0 || e >= p.cap) e = -1;
            if (e < 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) h[i] = 0;
            } else {
                const int64_t erow = uk.kv_row0 + e;
                const int d0 = c * 16;
                if (d0 < dn) {
                    const uint4 cv = __ldg(reinterpret_cast<const uint4*>(p.codes + erow * dn + d0));
                    const float sc = __ldg(p.scales + erow * ng + d0 / p.g);
                    const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 a = unpack_half2(e4m3x2_to_f16x2(static_cast<uint16_t>(cw[i] & 0xFFFFu)));
                        const float2 b = unpack_half2(e4m3x2_to_f16x2(static_cast<uint16_t>(cw[i] >> 16)));
                        h[2 * i] = pack_half2(a.x * sc, a.y * sc);
                        h[2 * i + 1] = pack_half2(b.x * sc, b.y * sc);
                    }
                } else {
                    const uint4* rp = reinterpret_cast<const uint4*>(p.rope + erow * p.d_rope + (d0 - dn));
                    const uint4 v0 = __ldg(rp), v1 = __ldg(rp + 1);
                    const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        h[i] = pack_half2(__uint_as_float(vw[i] << 16), __uint_as_float(vw[i] & 0xFFFF0000u));
                }
            }
        } else if (slot < uk.n_c + uk.n_w) {
            const uint4* rp = reinterpret_cast<const uint4*>(uk.wrow + static_cast<size_t>(slot - uk.n_c) * D + c * 16);
            const uint4 v0 = __ldg(rp), v1 = __ldg(rp + 1);
            const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
                h[i] = pack_half2(__uint_as_float(vw[i] << 16), __uint_as_float(vw[i] & 0xFFFF0000u));
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) h[i] = 0;
        }
        *reinterpret_cast<uint4*>(ks + swz<D>(r, 2 * c)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(ks + swz<D>(r, 2 * c + 1)) = make_uint4(h[4], h[5], h[6], h[7]);
    }
}

template <int D, int HP>
__global__ void __launch_bounds__(Cfg<D, HP>::NTHREADS, 1)
attn_kernel(Params p) {
    using C = Cfg<D, HP>;
    extern __shared__ __align__(128) char smem[];
    char* qs = smem;
    char* ks = smem + C::Q_BYTES;
    float* xs = reinterpret_cast<float*>(smem + C::Q_BYTES + C::K_BYTES);
    const uint32_t qs_a = static_cast<uint32_t>(__cvta_generic_to_shared(qs));
    const uint32_t ks_a = static_cast<uint32_t>(__cvta_generic_to_shared(ks));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hg = warp % C::NHG, half = warp / C::NHG;
    const int64_t u = blockIdx.x;
    const int split = blockIdx.y;
    const UnitKeys uk = unit_keys(p, u, D);
    const int n_tot = uk.n_c + uk.n_w;
    const int n_tiles = (n_tot + TK - 1) / TK;
    const int t_begin = split * p.tiles_per_split;
    const int t_end = min(n_tiles, t_begin + p.tiles_per_split);

    __shared__ float s_qr[HP];
    __shared__ float s_cos[32], s_sin[32];
    const bool q_extras = p.q_norm_w != nullptr || p.inv_freq != nullptr;
    if (q_extras) {
        // section 9 extras of the query: 1 / rms per head (partial sums of squares
        // per 16-byte vector in the exchange buffer, free until the first tile),
        // the RoPE table of the unit's position
        if (p.inv_freq && tid < p.d_rope / 2) rope_cs(p.inv_freq, tid, unit_pos(p, u), s_cos[tid], s_sin[tid]);
        if (p.q_norm_w) {
            for (int w = tid; w < HP * (D / 8); w += C::NTHREADS) {
                const int r = w / (D / 8), c = w % (D / 8);
                float ss = 0.0f;
                if (r < p.H) {
                    const uint4 b = __ldg(reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(u) * p.H + r) * D + c * 8));
                    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float x0 = __uint_as_float(bw[i] << 16), x1 = __uint_as_float(bw[i] & 0xFFFF0000u);
                        ss += x0 * x0 + x1 * x1;
                    }
                }
                xs[w] = ss;
            }
            __syncthreads();
            if (tid < HP) {
                float ss = 0.0f;
                for (int c = 0; c < D / 8; ++c) ss += xs[tid * (D / 8) + c];
                s_qr[tid] = rsqrtf(ss / static_cast<float>(D) + p.norm_eps);
            }
        }
        __syncthreads();
    }
    // Q -> fp16 (rows >= H zero)
    for (int w = tid; w < HP * (D / 8); w += C::NTHREADS) {
        const int r = w / (D / 8), c = w % (D / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < p.H) {
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(u) * p.H + r) * D + c * 8));
            const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) { f[2 * i] = __uint_as_float(bw[i] << 16); f[2 * i + 1] = __uint_as_float(bw[i] & 0xFFFF0000u); }
            if (p.q_norm_w) {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = f[i] * s_qr[r] * __ldg(p.q_norm_w + c * 8 + i);
            }
            if (p.inv_freq && c * 8 >= D - p.d_rope) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pi = (c * 8 - (D - p.d_rope)) / 2 + i;
                    const float a = f[2 * i], bb = f[2 * i + 1];
                    f[2 * i] = a * s_cos[pi] - bb * s_sin[pi];
                    f[2 * i + 1] = a * s_sin[pi] + bb * s_cos[pi];
                }
            }
            v = make_uint4(pack_half2(f[0], f[1]), pack_half2(f[2], f[3]), pack_half2(f[4], f[5]), pack_half2(f[6], f[7]));
        }
        *reinterpret_cast<uint4*>(qs + swz<D>(r, c)) = v;
    }

    float o[C::NT_O][4];
#pragma unroll
    for (int j = 0; j < C::NT_O; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.0f, 0.0f};

    const int g8 = lane >> 2, q4 = lane & 3;
    for (int t = t_begin; t < t_end; ++t) {
        __syncthreads();
        load_tile<D, C::NTHREADS>(p, uk, t * TK, ks);
        __syncthreads();

        // ---- partial S = Q[hg rows, half dims] . K[tile, half dims]^T
        float s[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.0f;
#pragma unroll 4
        for (int kk = 0; kk < C::KS_QK; ++kk) {
            const int chunk0 = (half * C::DH) / 8 + kk * 2;
            uint32_t a[4];
            {
                const int row = hg * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                ldsm_x4(qs_a + swz<D>(row, chunk0 + (lane >> 4)), a);
            }
#pragma unroll
            for (int nt = 0; nt < 8; nt += 2) {
                uint32_t b[4];
                const int mi = lane >> 3;
                const int key = nt * 8 + (lane & 7) + 8 * (mi >> 1);
                ldsm_x4(ks_a + swz<D>(key, chunk0 + (mi & 1)), b);
                mma16816(s[nt], a, b[0], b[1]);
                mma16816(s[nt + 1], a, b[2], b[3]);
            }
        }
        // ---- exchange partial sums between the two halves (fixed order: half 0 + half 1)
        float* mine = xs + static_cast<size_t>(warp) * 32 * 32;
        const int partner = hg + (1 - half) * C::NHG;
        const float* other = xs + static_cast<size_t>(partner) * 32 * 32;
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) mine[(j * 4 + i) * 32 + lane] = s[j][i];
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float x = other[(j * 4 + i) * 32 + lane];
                s[j][i] = half == 0 ? s[j][i] + x : x + s[j][i];
            }

        // ---- online softmax (base-2 logits), rows g8 and g8+8 of this head group
        const int slot0 = t * TK;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int key = slot0 + j * 8 + q4 * 2 + (i & 1);
                const float v = key < n_tot ? s[j][i] * p.scale_log2 : -INFINITY;
                s[j][i] = v;
                mx[i >> 1] = fmaxf(mx[i >> 1], v);
            }
        }
        float alpha[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            const float mn = fmaxf(m_r[r], mx[r]);
            alpha[r] = (mn == -INFINITY) ? 1.0f : exp2f(m_r[r] - mn);
            m_r[r] = mn;
        }
        float rs[2] = {0.0f, 0.0f};
        uint32_t pa[8][2];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float e[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float mr = m_r[i >> 1];
                e[i] = (mr == -INFINITY) ? 0.0f : exp2f(s[j][i] - mr);
            }
            pa[j][0] = pack_half2(e[0], e[1]);
            pa[j][1] = pack_half2(e[2], e[3]);
            const float2 r0 = unpack_half2(pa[j][0]), r1 = unpack_half2(pa[j][1]);
            rs[0] += r0.x + r0.y;
            rs[1] += r1.x + r1.y;
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
            rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
            l_r[r] = l_r[r] * alpha[r] + rs[r];
        }
#pragma unroll
        for (int j = 0; j < C::NT_O; ++j) {
            o[j][0] *= alpha[0]; o[j][1] *= alpha[0];
            o[j][2] *= alpha[1]; o[j][3] *= alpha[1];
        }
        // ---- O[hg rows, half dims] += P . V   (V = the same tile)
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
            const uint32_t a[4] = {pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1]};
            const int mi = lane >> 3;
            const int key = kk * 16 + (lane & 7) + 8 * (mi & 1);
#pragma unroll
            for (int nt = 0; nt < C::NT_O; nt += 2) {
                uint32_t b[4];
                const int chunk = (half * C::DH) / 8 + nt + (mi >> 1);
                ldsm_x4_t(ks_a + swz<D>(key, chunk), b);
                mma16816(o[nt], a, b[0], b[1]);
                mma16816(o[nt + 1], a, b[2], b[3]);
            }
        }
    }

    // ---- epilogue
    const int h0 = hg * 16 + g8, h1 = h0 + 8;
    const size_t ou = static_cast<size_t>(u);
    if (p.n_splits == 1) {
        // the sink joins the denominator (relative to the running max)
        float lt[2] = {l_r[0], l_r[1]};
        if (p.sink) {
            if (lt[0] > 0.0f && h0 < p.H) lt[0] += exp2f(__ldg(p.sink + h0) * LOG2E - m_r[0]);
            if (lt[1] > 0.0f && h1 < p.H) lt[1] += exp2f(__ldg(p.sink + h1) * LOG2E - m_r[1]);
        }
        const float inv0 = lt[0] > 0.0f ? 1.0f / lt[0] : 0.0f;
        const float inv1 = lt[1] > 0.0f ? 1.0f / lt[1] : 0.0f;
#pragma unroll
        for (int j = 0; j < C::NT_O; ++j) {
            const int col = half * C::DH + j * 8 + q4 * 2;
            float v0 = o[j][0] * inv0, v1 = o[j][1] * inv0, v2 = o[j][2] * inv1, v3 = o[j][3] * inv1;
            if (p.inv_freq && col >= D - p.d_rope) {
                // RoPE dims: rotate the output back by the query's position
                const int pi = (col - (D - p.d_rope)) / 2;
                const float cs = s_cos[pi], sn = s_sin[pi];
                const float a0 = v0 * cs + v1 * sn, a1 = v1 * cs - v0 * sn;
                const float b0 = v2 * cs + v3 * sn, b1 = v3 * cs - v2 * sn;
                v0 = a0; v1 = a1; v2 = b0; v3 = b1;
            }
            if (h0 < p.H) {
                __nv_bfloat162 v = __floats2bfloat162_rn(v0, v1);
                *reinterpret_cast<__nv_bfloat162*>(p.out + (ou * p.H + h0) * D + col) = v;
            }
            if (h1 < p.H) {
                __nv_bfloat162 v = __floats2bfloat162_rn(v2, v3);
                *reinterpret_cast<__nv_bfloat162*>(p.out + (ou * p.H + h1) * D + col) = v;
            }
        }
        if (p.lse && half == 0 && q4 == 0) {
            const float ln2 = 0.69314718055994531f;
            if (h0 < p.H)
                p.lse[ou * p.H + h0] = lt[0] > 0.0f ? (m_r[0] + log2f(lt[0])) * ln2 : (p.sink ? __ldg(p.sink + h0) : -INFINITY);
            if (h1 < p.H)
                p.lse[ou * p.H + h1] = lt[1] > 0.0f ? (m_r[1] + log2f(lt[1])) * ln2 : (p.sink ? __ldg(p.sink + h1) : -INFINITY);
        }
    } else {
        const size_t ps = ou * p.n_splits + split;
        float* po = p.part_o + ps * HP * D;
#pragma unroll
        for (int j = 0; j < C::NT_O; ++j) {
            const int col = half * C::DH + j * 8 + q4 * 2;
            *reinterpret_cast<float2*>(po + static_cast<size_t>(h0) * D + col) = make_float2(o[j][0], o[j][1]);
            *reinterpret_cast<float2*>(po + static_cast<size_t>(h1) * D + col) = make_float2(o[j][2], o[j][3]);
        }
        if (half == 0 && q4 == 0) {
            float* ml = p.part_ml + ps * 2 * HP;
            ml[h0] = m_r[0]; ml[HP + h0] = l_r[0];
            ml[h1] = m_r[1]; ml[HP + h1] = l_r[1];
        }
    }
}

// Log-sum-exp combine of the split partials: one block per (unit, head),
// D/4 threads, 4 dims each.
template <int D, int HP>
__global__ void combine_kernel(Params p) {
    const int64_t u = blockIdx.x;
    const int h = blockIdx.y;
    const int S = p.n_splits;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, p.part_ml[((u * S + s) * 2) * HP + h]);
    float L = 0.0f;
    float acc[4] = {0, 0, 0, 0};
    const int d0 = threadIdx.x * 4;
    for (int s = 0; s < S; ++s) {
        const float* ml = p.part_ml + ((u * S + s) * 2) * HP;
        const float ms = ml[h], ls = ml[HP + h];
        if (ls <= 0.0f || ms == -INFINITY) continue;
        const float wgt = exp2f(ms - M);
        L += wgt * ls;
        const float4 v = *reinterpret_cast<const float4*>(p.part_o + ((u * S + s) * HP + h) * static_cast<size_t>(D) + d0);
        acc[0] += wgt * v.x; acc[1] += wgt * v.y; acc[2] += wgt * v.z; acc[3] += wgt * v.w;
    }
    const float sink = p.sink ? __ldg(p.sink + h) : -INFINITY;
    if (p.sink && L > 0.0f) L += exp2f(sink * LOG2E - M);      // the sink joins the denominator
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    float o[4] = {acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv};
    if (p.inv_freq && d0 >= D - p.d_rope) {
        // RoPE dims: rotate the output back by the query's position
        const int64_t t = unit_pos(p, u);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float cs, sn;
            rope_cs(p.inv_freq, (d0 - (D - p.d_rope)) / 2 + i, t, cs, sn);
            const float x = o[2 * i], y = o[2 * i + 1];
            o[2 * i] = x * cs + y * sn;
            o[2 * i + 1] = y * cs - x * sn;
        }
    }
    __nv_bfloat162 a = __floats2bfloat162_rn(o[0], o[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(o[2], o[3]);
    uint2 w;
    w.x = *reinterpret_cast<uint32_t*>(&a);
    w.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p.out + (static_cast<size_t>(u) * p.H + h) * D + d0) = w;
    if (p.lse && threadIdx.x == 0)
        p.lse[u * p.H + h] = L > 0.0f ? (M + log2f(L)) * 0.69314718055994531f : sink;
}

}  // namespace attn

namespace {

template <int D, int HP>
int launch_attn(attn::Params& p, int64_t units, cudaStream_t st) {
    using C = attn::Cfg<D, HP>;
    cudaError_t e = cudaFuncSetAttribute(attn::attn_kernel<D, HP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(C::SMEM));
    if (e != cudaSuccess) { set_last_cuda_error(static_cast<int>(e)); return HCA_ERR_CUDA; }
    attn::attn_kernel<D, HP><<<dim3(static_cast<unsigned>(units), p.n_splits), C::NTHREADS, C::SMEM, st>>>(p);
    HCA_CHECK_LAUNCH();
    if (p.n_splits > 1) {
        attn::combine_kernel<D, HP><<<dim3(static_cast<unsigned>(units), p.H), D / 4, 0, st>>>(p);
        HCA_CHECK_LAUNCH();
    }
    return HCA_OK;
}

int dispatch(attn::Params& p, int D, int64_t units, cudaStream_t st) {
    if (D == 512 && p.H == 64) return launch_attn<512, 64>(p, units, st);
    if (D == 128 && p.H == 64) return launch_attn<128, 64>(p, units, st);
    if (D == 128 && p.H <= 16) return launch_attn<128, 16>(p, units, st);
    return HCA_ERR_UNSUPPORTED;
}

int heads_padded(int D, int H) { return (D == 128 && H <= 16) ? 16 : 64; }

}  // namespace

// tensor-core (tcgen05) path for d = 512, H = 64: attention_tc.cu
void tc_decode_plan(int B, int max_comp, int W, bool sparse, int& n_splits, int& tiles_per_split);
size_t tc_decode_ws_bytes(int B, int max_comp, int W, bool sparse);
int tc_attn_decode_launch(const uint16_t* q, int B, int H, const hca_kv_cache& kv, const int32_t* idx,
                          int idx_stride, const int32_t* n_comp, int max_comp, const uint16_t* window, int W,
                          float softmax_scale, const hca_attn_extras* ex, uint16_t* out, float* lse, void* ws,
                          size_t ws_bytes, cudaStream_t st);
int tc_attn_prefill_launch(const uint16_t* q, int Tq, int H, int p0, int m, const hca_kv_cache& kv,
                           const int32_t* idx, int idx_stride, const int32_t* count, const uint16_t* raw, int W,
                           float softmax_scale, const hca_attn_extras* ex, uint16_t* out, cudaStream_t st);

static void set_extras(attn::Params& p, const hca_attn_extras* ex, bool decode) {
    if (!ex) return;
    p.q_norm_w = ex->q_norm_w;
    p.norm_eps = ex->norm_eps;
    p.sink = ex->sink;
    p.inv_freq = ex->inv_freq;
    p.q_pos = decode ? ex->q_pos : nullptr;
    p.win_len = decode ? ex->win_len : nullptr;
}
static bool use_tc(int D, int H) { return D == 512 && H == 64; }

// split-K plan shared by the workspace query and the launch
void decode_plan(int B, int max_comp, int W, int& n_splits, int& tiles_per_split) {
    const int n_tiles = static_cast<int>(ceil_div(static_cast<int64_t>(max_comp) + W, attn::TK));
    int splits = sm_count() / (B > 0 ? B : 1);
    if (splits < 1) splits = 1;
    if (splits > n_tiles) splits = n_tiles > 0 ? n_tiles : 1;
    tiles_per_split = static_cast<int>(ceil_div(n_tiles > 0 ? n_tiles : 1, splits));
    n_splits = static_cast<int>(ceil_div(n_tiles > 0 ? n_tiles : 1, tiles_per_split));
}

size_t decode_ws_bytes(int B, int H, int D, int max_comp, int W) {
    if (use_tc(D, H)) {
        const size_t a = tc_decode_ws_bytes(B, max_comp, W, true), b = tc_decode_ws_bytes(B, max_comp, W, false);
        return a > b ? a : b;
    }
    int ns, tps;
    decode_plan(B, max_comp, W, ns, tps);
    if (ns <= 1) return 0;
    const int HP = heads_padded(D, H);
    return static_cast<size_t>(B) * ns * HP * (static_cast<size_t>(D) + 2) * sizeof(float) + 256;
}

int attn_decode_launch(const uint16_t* q, int B, int H, const hca_kv_layout& L, const hca_kv_cache& kv,
                       const int32_t* idx, int idx_stride, const int32_t* n_comp, int max_comp,
                       const uint16_t* window, int W, float softmax_scale, const hca_attn_extras* ex,
                       uint16_t* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t st) {
    if (!(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return HCA_ERR_INVALID_ARG;
    if (B == 0) return HCA_OK;
    if (use_tc(L.d, H))
        return tc_attn_decode_launch(q, B, H, kv, idx, idx_stride, n_comp, max_comp, window, W, softmax_scale, ex,
                                     out, lse, ws, ws_bytes, st);
    attn::Params p = {};
    set_extras(p, ex, true);
    p.q = q; p.H = H;
    p.codes = kv.codes; p.scales = kv.scales; p.rope = kv.rope; p.cap = kv.capacity;
    p.d_rope = L.d_rope; p.g = L.scale_group;
    p.prefill = 0;
    p.idx = idx; p.idx_stride = idx_stride; p.n_comp = n_comp;
    p.win = window; p.W = W;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    decode_plan(B, max_comp, W, p.n_splits, p.tiles_per_split);
    p.out = out; p.lse = lse;
    if (p.n_splits > 1) {
        const size_t need = decode_ws_bytes(B, H, L.d, max_comp, W);
        if (ws == nullptr || ws_bytes < need) return HCA_ERR_WORKSPACE;
        const int HP = heads_padded(L.d, H);
        p.part_o = reinterpret_cast<float*>(ws);
        p.part_ml = p.part_o + static_cast<size_t>(B) * p.n_splits * HP * L.d;
    }
    return dispatch(p, L.d, B, st);
}

int attn_prefill_launch(const uint16_t* q, int Tq, int H, int p0, int m, const hca_kv_layout& L,
                        const hca_kv_cache& kv, const int32_t* idx, int idx_stride, const int32_t* count,
                        const uint16_t* raw, int W, float softmax_scale, const hca_attn_extras* ex, uint16_t* out,
                        cudaStream_t st) {
    if (!(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return HCA_ERR_INVALID_ARG;
    if (Tq == 0) return HCA_OK;
    if (use_tc(L.d, H))
        return tc_attn_prefill_launch(q, Tq, H, p0, m, kv, idx, idx_stride, count, raw, W, softmax_scale, ex, out,
                                      st);
    attn::Params p = {};
    set_extras(p, ex, false);
    p.q = q; p.H = H;
    p.codes = kv.codes; p.scales = kv.scales; p.rope = kv.rope; p.cap = kv.capacity;
    p.d_rope = L.d_rope; p.g = L.scale_group;
    p.prefill = 1;
    p.idx = idx; p.idx_stride = idx_stride; p.n_comp = count;
    p.dense_m = m; p.p0 = p0;
    p.win = raw; p.W = W;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.n_splits = 1;
    p.tiles_per_split = 1 << 30;
    p.out = out; p.lse = nullptr;
    return dispatch(p, L.d, Tq, st);
}

// ------------------------------------------------------------------
// Decode attention without a caller workspace.
//
// For callers that cannot allocate device memory when they call us (a
// plug-in inside an engine that owns all device memory and allows no
// allocation after start-up; a latency-critical path that cannot afford
// cudaMalloc's implicit synchronisation), the split-K partials live in this
// file-scope array instead of a caller buffer.  The array is a global of the
// loaded library, so every device it runs on keeps HCA_NOALLOC_SCRATCH_BYTES
// until the process exits.  Host code must not pass `g_noalloc_scratch`
// itself to a kernel: in host code that name is only a host-side stand-in.
// Every call looks up the device address of the array for the current
// device with cudaGetSymbolAddress (cheap; nothing is allocated), so an
// address never outlives the context it came from.  The first call on a
// device also loads the library's device globals there, so it should come
// before any stream capture.  All calls on a device share the array; the
// kernels write every partial before reading it, so no clearing is needed,
// but calls that overlap on the GPU race on it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HCA_NOALLOC_SCRATCH_BYTES];

namespace {

void* noalloc_scratch_address(int* status) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
        set_last_cuda_error(static_cast<int>(e));
        *status = HCA_ERR_CUDA;
        return nullptr;
    }
    *status = HCA_OK;
    return p;
}

bool noalloc_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace hca

extern "C" int compressed_attn_decode_noalloc(const uint16_t* q, int32_t B, int32_t H, hca_kv_layout layout,
                                              hca_kv_cache kv, const int32_t* idx, int32_t idx_stride,
                                              const int32_t* n_comp, int32_t max_comp, const uint16_t* window,
                                              int32_t W, float softmax_scale, uint16_t* out, float* lse,
                                              void* stream) {
    using namespace hca;
    // the same argument rules as compressed_attn_decode
    if (!(B >= 0 && max_comp >= 0 && W >= 0)) return HCA_ERR_INVALID_ARG;
    const bool layout_ok = (layout.d == 512 && layout.d_rope == 64 && layout.scale_group == 64) ||
                           (layout.d == 128 && layout.d_rope == 32 && layout.scale_group == 32);
    if (!layout_ok) return HCA_ERR_UNSUPPORTED;
    if (!((layout.d == 512 && H == 64) || (layout.d == 128 && (H == 64 || (H >= 1 && H <= 16)))))
        return HCA_ERR_UNSUPPORTED;
    if (W > 4096) return HCA_ERR_UNSUPPORTED;
    if (B == 0) return HCA_OK;
    if (!q || !noalloc_aligned16(q) || !n_comp || !noalloc_aligned16(n_comp) || !out || !noalloc_aligned16(out))
        return HCA_ERR_INVALID_ARG;
    if (!kv.codes || !kv.scales || !kv.rope || !noalloc_aligned16(kv.codes) || !noalloc_aligned16(kv.scales) ||
        !noalloc_aligned16(kv.rope) || kv.capacity < 0)
        return HCA_ERR_INVALID_ARG;
    if (W > 0 && (!window || !noalloc_aligned16(window))) return HCA_ERR_INVALID_ARG;
    if (idx && (!noalloc_aligned16(idx) || idx_stride < max_comp)) return HCA_ERR_INVALID_ARG;
    if (lse && !noalloc_aligned16(lse)) return HCA_ERR_INVALID_ARG;
    const size_t need = decode_ws_bytes(B, H, layout.d, max_comp, W);
    if (need > HCA_NOALLOC_SCRATCH_BYTES) return HCA_ERR_SCRATCH_LIMIT;
    int st = HCA_OK;
    void* scratch = noalloc_scratch_address(&st);
    if (st != HCA_OK) return st;
    return attn_decode_launch(q, B, H, layout, kv, idx, idx_stride, n_comp, max_comp, window, W, softmax_scale,
                              nullptr, out, lse, scratch, HCA_NOALLOC_SCRATCH_BYTES, as_stream(stream));
}
