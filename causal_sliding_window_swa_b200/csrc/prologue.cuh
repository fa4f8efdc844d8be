// prologue.cuh -- the HBM-bound steps before the attention product:
//   * RoPE on q and k, then parameter-free RMS normalisation (intelliparadigm "GPT-2 for $73",
//     section 2.2: q, k = norm(rope(q)), norm(rope(k)); section 2.1: RMSNorm without gamma/beta);
//   * the gated value embedding v' = v + 2 sigmoid(x[..., :32] . Wg[:, h]) * ve (PaperWeekly
//     repost, "Value Embeddings" paragraph), one gate per (b, t, h).
// Pair layout of the rotation: (i, i + D/2), theta_i = base^(-2i/D), position t rotates
// (a, b) -> (a cos - b sin, a sin + b cos).
//
// Rounding.  Every output element is the correctly rounded bf16 (nearest, ties to even) of the
// exact value of its definition, so the tensor-core operands do not depend on how the arithmetic
// is organised (an fp32-only pipeline flips the last bf16 bit of ~1e-4 of the elements, which
// moves single attention scores by ~1e-3).  The common path runs in fp32 with a proven error
// bound; an element whose fp32 result could round differently from the exact one (a few in 10^4)
// is listed, and its block recomputes it in fp64 and overwrites it after its last row chunk.
//   norm: r = 1 / sqrt(ss / D + eps) from the sum of squares of the raw inputs (the rotation
//     preserves it) in fp64, where each square and the sum are exact; the inverse square root by
//     two Newton-Raphson steps from the hardware estimate, then rounded once to fp32.
//   rotation: cos and sin are stored as a head with a 16-bit significand, so that a * head is
//     exact in fp32 for a bf16 input a, and the fp32 remainder (|c - head - tail| < 2^-40).  With
//     S = |a| + |b|: the head term a c_hi - b s_hi is one fma of exact operands (error 2^-24 of
//     itself), the tail term costs at most 2^-39 S, the table 2^-40 S, so ra is within
//     2^-23 |ra| + 2^-38 S of the exact rotation and x = ra * r within 2^-22 |x| + 2^-38 S r, i.e.
//     within 5 of its own ulps whenever |x| >= 2^-14 S r.  The test window is 8 ulps, and smaller
//     |x| (partial cancellation, a few in 10^5 elements) always take the fp64 path.
//   gate: z = x[:32] . Wg[:, h] and g = 2 sigmoid(z) in fp64 by a separate one-thread-per-row
//     kernel, stored split as g_hi + g_lo (fp32); v' = (v + g_hi ve) + g_lo ve with two fp32
//     roundings: within 1 ulp of the exact value unless |v'| < 2^-16 |g ve|.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace swa {

// Division by a loop-invariant divisor d for 0 <= n < 2^31: q = (n * m) >> k with
// k = 32 + ceil(log2 d) and m = ceil(2^k / d) (Granlund and Montgomery, "Division by invariant
// integers using multiplication", 1994: the error term n (m d - 2^k) / (d 2^k) stays below 1/d).
struct FastDiv {
    unsigned long long m;
    int k;
    int d;
};

__device__ __forceinline__ int fdiv(int n, const FastDiv& f) {
    return (int)(((unsigned long long)(unsigned)n * f.m) >> f.k);
}

// Gate of every (b, t, h) row: g = 2 sigmoid(sum_{c<32} x[b,t,c] Wg[c,h]) in fp64, stored as
// (g_hi, g_lo) = (fp32(g), fp32(g - g_hi)) at gate[bt * H + h].  One thread per token bt: its 32
// gate channels (at gate_x + bt * x_stride: 32 for the contiguous slice, C for the full layer
// input) are loaded once, and the heads are taken four at a time, each sum over c in order.  Wg
// (32 x H) is staged in shared memory as fp64 (32 H doubles of dynamic shared memory) when
// wg_smem is set, else read from global memory.
__global__ void gate_kernel(const __nv_bfloat16* __restrict__ gate_x, const __nv_bfloat16* __restrict__ Wg,
                            float2* __restrict__ gate, int n_tokens, int H, int x_stride, int wg_smem) {
    extern __shared__ double s_wg[];   // [32][H]
    grid_dependents_launch();          // the prologue kernel may launch (it waits for this one)
    if (wg_smem)
        for (int i = threadIdx.x; i < 32 * H; i += blockDim.x) s_wg[i] = (double)__bfloat162float(Wg[i]);
    __syncthreads();
    auto wg = [&](int i) -> double { return wg_smem ? s_wg[i] : (double)__bfloat162float(Wg[i]); };
    for (int bt = blockIdx.x * blockDim.x + threadIdx.x; bt < n_tokens; bt += gridDim.x * blockDim.x) {
        const __nv_bfloat16* xr = gate_x + (long long)bt * x_stride;
        double x[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] = (double)__bfloat162float(xr[c]);
        for (int h0 = 0; h0 < H; h0 += 4) {
            double z[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
            for (int c = 0; c < 32; ++c)
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (h0 + u < H) z[u] = fma(x[c], wg(c * H + h0 + u), z[u]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (h0 + u >= H) break;
                const double g = 2.0 / (1.0 + exp(-z[u]));
                const float g_hi = (float)g;
                gate[(long long)bt * H + h0 + u] = make_float2(g_hi, (float)(g - (double)g_hi));
            }
        }
    }
}

// RoPE tables, one entry per (t, i):
//   tab32[t*D/2 + i] = (c_hi, c_lo, s_hi, s_lo) fp32: c_hi with a 16-bit significand, c_lo the
//     fp32 of the remainder c - c_hi (likewise s);
//   tab64[t*D/2 + i] = (cos, sin) fp64, read only by the fp64 path.
__device__ __forceinline__ float round_sig16(double x) {
    // nearest float with at most 16 significant bits (8 low mantissa bits cleared)
    const float f = (float)x;
    const uint32_t u = __float_as_uint(f);
    return __uint_as_float((u + 0x80u) & 0xffffff00u);
}

// c -> (hi, lo): hi = c to 16 significant bits, lo = fp32(c - hi); |c - hi - lo| <= 2^-40 |c|.
__device__ __forceinline__ void rope_split(double c, float& hi, float& lo) {
    hi = round_sig16(c);
    lo = (float)(c - (double)hi);
}

// tab2 (optional, for the fused projection's epilogue): (c_hi + c_lo, s_hi + s_lo) summed in fp32,
// the values that epilogue uses; tab64 may then be null (the fused path keeps tab2 in its place).
__global__ void rope_table_kernel(float4* __restrict__ tab32, double2* __restrict__ tab64, float2* __restrict__ tab2,
                                  int T, int D, double base) {
    const int half = D / 2;
    const long long n = (long long)T * half;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(idx / half);
        const int i = (int)(idx % half);
        const double theta = pow(base, -2.0 * (double)i / (double)D);
        double s, c;
        sincos((double)t * theta, &s, &c);
        float c_hi, c_lo, s_hi, s_lo;
        rope_split(c, c_hi, c_lo);
        rope_split(s, s_hi, s_lo);
        tab32[idx] = make_float4(c_hi, c_lo, s_hi, s_lo);
        if (tab64 != nullptr) tab64[idx] = make_double2(c, s);
        if (tab2 != nullptr) tab2[idx] = make_float2(c_hi + c_lo, s_hi + s_lo);
    }
}

__device__ __forceinline__ uint2 ldg_stream8(const void* p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void unpack4(const uint2& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xffff0000u);
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint16_t bf16_rn_bits(double x) {
    return __bfloat16_as_ushort(__double2bfloat16(x));
}

// 1 / sqrt(y) for y > 0 in fp64: the hardware fp32 estimate refined by two Newton-Raphson steps
// for the inverse square root, r <- r (3 - y r^2) / 2 (each step squares the relative error:
// ~2^-22 -> 2^-44 -> below 2^-52).
__device__ __forceinline__ double rsqrt_newton(double y) {
    double r = (double)rsqrtf((float)y);
    r = r * fma(-0.5 * y, r * r, 1.5);
    r = r * fma(-0.5 * y, r * r, 1.5);
    return r;
}

// True if the low 16 bits of x are within 8 of 0x8000: a bf16 rounding midpoint lies within
// [-8, +7] fp32 ulps of x.
__device__ __forceinline__ bool near_midpoint_8ulp(float x) {
    return ((__float_as_uint(x) + 8u - 0x8000u) & 0xfff0u) == 0u;
}

// Fast path of four rotation pairs (a_e, b_e) = (element i0 + e, element i0 + e + D/2) of one
// row, scaled by r: the bf16 words of (a'_0..a'_3) and (b'_0..b'_3) rounded from fp32, and a mask
// with bit e set where pair e could round differently from its exact value (near a bf16 rounding
// midpoint, or partial cancellation).  No branch: the caller repairs masked pairs afterwards.
__device__ __forceinline__ uint32_t rope_rms_fast4(const float (&a)[4], const float (&b)[4], const float4 (&w)[4],
                                                   float r, uint2& out_lo, uint2& out_hi) {
    float xa[4], xb[4];
    uint32_t mask = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        // head products are exact (one rounding per head fma); tail terms are 2^-16 smaller
        const float ra = fmaf(a[e], w[e].x, -(b[e] * w[e].z)) + fmaf(a[e], w[e].y, -(b[e] * w[e].w));
        const float rb = fmaf(a[e], w[e].z, b[e] * w[e].x) + fmaf(a[e], w[e].w, b[e] * w[e].y);
        xa[e] = ra * r;
        xb[e] = rb * r;
        const float small = r * (fabsf(a[e]) + fabsf(b[e])) * 0x1p-14f;
        const bool slow = near_midpoint_8ulp(xa[e]) | near_midpoint_8ulp(xb[e]) | (fabsf(xa[e]) < small) |
                          (fabsf(xb[e]) < small);
        mask |= (slow ? 1u : 0u) << e;
    }
    out_lo = make_uint2(pack_bf16x2(xa[0], xa[1]), pack_bf16x2(xa[2], xa[3]));
    out_hi = make_uint2(pack_bf16x2(xb[0], xb[1]), pack_bf16x2(xb[2], xb[3]));
    return mask;
}

// Replaces 16-bit element e (0..3) of a 4-element bf16 word pair.
__device__ __forceinline__ void set_bf16_elem(uint2& w, int e, uint16_t v) {
    uint32_t& word = (e >> 1) ? w.y : w.x;
    word = (e & 1) ? ((word & 0x0000ffffu) | ((uint32_t)v << 16)) : ((word & 0xffff0000u) | v);
}

// The masked pairs of rope_rms_fast4 in fp64, rounded once: ((a cos - b sin) r64, (a sin + b cos) r64).
__device__ __noinline__ void rope_rms_repair4(const float (&a)[4], const float (&b)[4], const double2* __restrict__ t64,
                                              double r64, uint32_t mask, uint2& out_lo, uint2& out_hi) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if (!((mask >> e) & 1u)) continue;
        const double2 tw = t64[e];
        const double Ad = (double)a[e], Bd = (double)b[e];
        set_bf16_elem(out_lo, e, bf16_rn_bits((Ad * tw.x - Bd * tw.y) * r64));
        set_bf16_elem(out_hi, e, bf16_rn_bits((Ad * tw.y + Bd * tw.x) * r64));
    }
}

// One group of D/8 consecutive threads handles one (b, t, h) row.  Thread c of the group owns
// pairs i in [4c, 4c+4): elements i (in `lo_raw`) and i + D/2 (in `hi_raw`).  Returns the mask of
// pairs still to be repaired (rope_rms_repair4 with the returned r64).
template <int D>
__device__ __forceinline__ uint32_t rope_rms_pairs4(const uint2& lo_raw, const uint2& hi_raw, const float4 (&cs)[4],
                                                    double eps, float (&a)[4], float (&b)[4], uint2& out_lo,
                                                    uint2& out_hi, double& r64) {
    constexpr int TPR = D / 8;
    unpack4(lo_raw, a);
    unpack4(hi_raw, b);
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        ss = fma((double)a[e], (double)a[e], ss);
        ss = fma((double)b[e], (double)b[e], ss);
    }
#pragma unroll
    for (int m = TPR / 2; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    r64 = rsqrt_newton(ss * (1.0 / (double)D) + eps);
    return rope_rms_fast4(a, b, cs, (float)r64, out_lo, out_hi);
}

// v' = v + g ve for 4 elements: (v + g_hi ve) + g_lo ve in fp32 (two roundings, within 1 ulp
// unless |v'| < 2^-16 |g ve|).  Returns the mask of elements that could cross a bf16 rounding
// midpoint (repaired in fp64 by gated_repair4).
__device__ __forceinline__ uint32_t gated_fast4(const uint2& vw, const uint2& ew, float g_hi, float g_lo, uint2& out) {
    float v[4], e4[4];
    unpack4(vw, v);
    unpack4(ew, e4);
    float x[4];
    uint32_t mask = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[e] = fmaf(g_lo, e4[e], fmaf(g_hi, e4[e], v[e]));
        const bool slow = near_midpoint_8ulp(x[e]) | (fabsf(x[e]) < fabsf(g_hi * e4[e]) * 0x1p-16f);
        mask |= (slow ? 1u : 0u) << e;
    }
    out = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
    return mask;
}

__device__ __noinline__ void gated_repair4(const uint2& vw, const uint2& ew, double g64, uint32_t mask, uint2& out) {
    float v[4], e4[4];
    unpack4(vw, v);
    unpack4(ew, e4);
#pragma unroll
    for (int e = 0; e < 4; ++e)
        if ((mask >> e) & 1u) set_bf16_elem(out, e, bf16_rn_bits(fma(g64, (double)e4[e], (double)v[e])));
}

// The two steps together, for callers with few rows (the decode step).
template <int D>
__device__ __forceinline__ void rope_rms_exact4(const uint2& lo_raw, const uint2& hi_raw, const float4 (&cs)[4],
                                                const double2* __restrict__ t64, double eps, uint2& out_lo,
                                                uint2& out_hi) {
    float a[4], b[4];
    double r64;
    const uint32_t m = rope_rms_pairs4<D>(lo_raw, hi_raw, cs, eps, a, b, out_lo, out_hi, r64);
    if (m) rope_rms_repair4(a, b, t64, r64, m, out_lo, out_hi);
}

__device__ __forceinline__ uint2 gated_add4(const uint2& vw, const uint2& ew, float g_hi, float g_lo, double g64) {
    uint2 out;
    const uint32_t m = gated_fast4(vw, ew, g_hi, g_lo, out);
    if (m) gated_repair4(vw, ew, g64, m, out);
    return out;
}

// ------------------------------------------------------------------ deferred repairs
// The prologue kernel writes every output from its fp32 fast path.  A row chunk (D/8 threads per
// row; four rotation pairs and eight v' elements per thread) with elements that fast path cannot
// certify goes on its block's shared-memory list as (chunk, flags): flag bits 0-3 qhat pairs
// i0 + e (elements i0 + e and i0 + e + D/2), bits 4-7 khat pairs, bits 8-11 v' elements i0 + e,
// bits 12-15 v' elements i0 + D/2 + e.  The grid is a single wave of blocks, so each block
// repairs its list once, after its last chunk: its threads recompute the listed elements in fp64
// and overwrite them.  A block whose list overflows (inputs built to sit on rounding midpoints)
// recomputes every element of its row chunks instead.  An item carries the rows' fp64 r (the fast
// path already has it), so that a repair needs only the chunk's own inputs.
constexpr int kFixPerBlock = 1024;

struct __align__(16) FixItem {
    uint32_t chunk_lo;     // row chunk index, low 32 bits
    uint32_t code;         // flag bits | (chunk index >> 32) << 16
    uint32_t pad0, pad1;
    double rq, rk;         // r of the chunk's qhat row and khat row (fp64)
};

struct FixParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const __nv_bfloat16* ve;
    const float2* gate;
    __nv_bfloat16* qh;
    __nv_bfloat16* kh;
    __nv_bfloat16* vp;
    const double2* tab64;
    int T;
    int heads;                 // heads of the pass's rows (H, or Hkv for the key/value pass)
    double eps;
};

// 1 / sqrt(ss / D + eps) of one row in fp64: exact squares, fp64 sums.  All loads are issued
// before the arithmetic.
template <int D>
__device__ __forceinline__ double row_r64(const __nv_bfloat16* __restrict__ x, double eps) {
    uint4 u[D / 8];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) u[j] = *reinterpret_cast<const uint4*>(x + 8 * j);
    double s0 = 0.0, s1 = 0.0;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        float f[4], g[4];
        unpack4(make_uint2(u[j].x, u[j].y), f);
        unpack4(make_uint2(u[j].z, u[j].w), g);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            s0 = fma((double)f[e], (double)f[e], s0);
            s1 = fma((double)g[e], (double)g[e], s1);
        }
    }
    return rsqrt_newton((s0 + s1) * (1.0 / (double)D) + eps);
}

// The flagged elements of one row chunk in fp64, each rounded once: the rotation with the fp64
// table scaled by the row's r; v + g ve with g = g_hi + g_lo.  The loads of a tensor's row and of
// the chunk's four pairs are issued together.  Out of line: it runs for a few chunks in 10^4.
template <int D>
__device__ __noinline__ void prologue_fix_chunk(long long chunk, uint32_t flags, const FixParams& p,
                                                double rq, double rk, bool r_known) {
    constexpr int TPR = D / 8, HALF = D / 2;
    const uint32_t row = (uint32_t)(chunk / TPR);
    const int i0 = 4 * (int)(chunk % TPR);
    const long long base = (long long)row * D;
    const uint32_t t = (row / (uint32_t)p.heads) % (uint32_t)p.T;
    const double2* tw = p.tab64 + (long long)t * HALF + i0;
#pragma unroll 1
    for (int tensor = 0; tensor < 2; ++tensor) {
        const uint32_t m = (flags >> (4 * tensor)) & 15u;
        if (m == 0u) continue;
        const __nv_bfloat16* x = (tensor == 0 ? p.q : p.k) + base;
        __nv_bfloat16* dst = (tensor == 0 ? p.qh : p.kh) + base;
        double2 cs[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) cs[e] = tw[e];
        float a[4], b[4];
        unpack4(*reinterpret_cast<const uint2*>(x + i0), a);
        unpack4(*reinterpret_cast<const uint2*>(x + HALF + i0), b);
        const double r64 = r_known ? (tensor == 0 ? rq : rk) : row_r64<D>(x, p.eps);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (!((m >> e) & 1u)) continue;
            const double A = (double)a[e], B = (double)b[e];
            dst[i0 + e] = __ushort_as_bfloat16(bf16_rn_bits((A * cs[e].x - B * cs[e].y) * r64));
            dst[HALF + i0 + e] = __ushort_as_bfloat16(bf16_rn_bits((A * cs[e].y + B * cs[e].x) * r64));
        }
    }
    const uint32_t mv = flags >> 8;
    if (mv != 0u) {
        const float2 g = p.gate[row];
        float v[8], e8[8];
        unpack4(*reinterpret_cast<const uint2*>(p.v + base + i0), *reinterpret_cast<float(*)[4]>(v));
        unpack4(*reinterpret_cast<const uint2*>(p.v + base + HALF + i0), *reinterpret_cast<float(*)[4]>(v + 4));
        unpack4(*reinterpret_cast<const uint2*>(p.ve + base + i0), *reinterpret_cast<float(*)[4]>(e8));
        unpack4(*reinterpret_cast<const uint2*>(p.ve + base + HALF + i0), *reinterpret_cast<float(*)[4]>(e8 + 4));
        const double g64 = (double)g.x + (double)g.y;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (!((mv >> e) & 1u)) continue;
            const int i = e < 4 ? i0 + e : HALF + i0 + e - 4;
            p.vp[base + i] = __ushort_as_bfloat16(bf16_rn_bits(fma(g64, (double)e8[e], (double)v[e])));
        }
    }
}

// PARTS selects the outputs: bit 0 qhat, bit 1 khat and v' (v' only on value-embedding layers).
// The multi-head layer runs both in one pass (PARTS = 3, rows (b,t,h) of all inputs); with
// grouped-query attention the query rows (H heads) and the key/value rows (Hkv heads) are two
// passes over their own row sets, `H` being that pass's head count.
template <int D, bool HAS_VE, int PARTS = 3>
__global__ void __launch_bounds__(256, 3) prologue_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ ve,
    const float2* __restrict__ gate,
    __nv_bfloat16* __restrict__ qh, __nv_bfloat16* __restrict__ kh, __nv_bfloat16* __restrict__ vp,
    const float4* __restrict__ tab32, const double2* __restrict__ tab64, int* __restrict__ sched,
    int n_rows, int T, int H, FastDiv divT, FastDiv divH, double eps) {
    constexpr int TPR = D / 8;           // threads per row (16 or 8); divides 32
    constexpr int LOG_TPR = (D == 128) ? 4 : 3;
    constexpr int HALF = D / 2;
    constexpr bool DO_Q = (PARTS & 1) != 0, DO_KV = (PARTS & 2) != 0;
    const long long gtid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
    // Every thread of a warp runs the same number of iterations, so the shuffles always see the
    // full warp; rows past the end are computed on zeros and not stored.
    const long long n_iter = ((long long)n_rows * TPR + stride - 1) / stride;
    // Launched as a programmatic dependent of the gate kernel: wait for it before any memory
    // access, then let the attention kernel launch (it waits for this grid to finish).
    grid_dependency_wait();
    grid_dependents_launch();
    // The attention kernel that follows takes its work items from this counter.
    if (gtid == 0) {
        sched[0] = 0;
        sched[1] = 0;
    }
    // This block's list of row chunks to repair once all of them are written.
    __shared__ int s_nfix;
    __shared__ FixItem s_fix[kFixPerBlock];
    if (threadIdx.x == 0) s_nfix = 0;
    __syncthreads();
    for (long long it = 0; it < n_iter; ++it) {
        const long long tid = gtid + it * stride;
        const int row_raw = (int)(tid >> LOG_TPR);           // (b*T + t)*H + h, < 2^31
        const int c = (int)(tid & (TPR - 1));
        const bool valid = row_raw < n_rows;
        const int row = valid ? row_raw : 0;
        const int bt = fdiv(row, divH);
        const int t = bt - fdiv(bt, divT) * T;
        const int i0 = 4 * c;
        const long long off = (long long)row * D;

        // Every load of this row chunk is issued before any arithmetic.
        uint2 raw[8];
        float2 gw = make_float2(0.f, 0.f);
        if (valid) {
            if (DO_Q) {
                raw[0] = ldg_stream8(q + off + i0);
                raw[1] = ldg_stream8(q + off + HALF + i0);
            }
            if (DO_KV) {
                raw[2] = ldg_stream8(k + off + i0);
                raw[3] = ldg_stream8(k + off + HALF + i0);
            }
            if (HAS_VE && DO_KV) {
                raw[4] = ldg_stream8(v + off + i0);
                raw[5] = ldg_stream8(v + off + HALF + i0);
                raw[6] = ldg_stream8(ve + off + i0);
                raw[7] = ldg_stream8(ve + off + HALF + i0);
                gw = __ldg(gate + row);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) raw[e] = make_uint2(0u, 0u);
        }
        if (!DO_Q) raw[0] = raw[1] = make_uint2(0u, 0u);
        if (!DO_KV || !HAS_VE)
#pragma unroll
            for (int e = 4; e < 8; ++e) raw[e] = make_uint2(0u, 0u);
        if (!DO_KV) raw[2] = raw[3] = make_uint2(0u, 0u);
        float4 cs[4];
        {
            const float4* tp = tab32 + (long long)t * HALF + i0;
#pragma unroll
            for (int e = 0; e < 4; ++e) cs[e] = __ldg(tp + e);
        }
        // Fast path for every output of the row chunk (one branch-free block); a chunk with
        // elements it cannot certify goes on the block's repair list.
        uint2 o0, o1, o2, o3, o4 = make_uint2(0u, 0u), o5 = make_uint2(0u, 0u);
        uint32_t mq = 0u, mk = 0u, mv = 0u;
        double rq = 0.0, rk = 0.0;
        {
            float a[4], b[4];
            if (DO_Q) mq = rope_rms_pairs4<D>(raw[0], raw[1], cs, eps, a, b, o0, o1, rq);
            if (DO_KV) mk = rope_rms_pairs4<D>(raw[2], raw[3], cs, eps, a, b, o2, o3, rk);
        }
        if (HAS_VE && DO_KV) {
            mv = gated_fast4(raw[4], raw[6], gw.x, gw.y, o4);
            mv |= gated_fast4(raw[5], raw[7], gw.x, gw.y, o5) << 4;
        }
        if (valid) {
            if (DO_Q) {
                *reinterpret_cast<uint2*>(qh + off + i0) = o0;
                *reinterpret_cast<uint2*>(qh + off + HALF + i0) = o1;
            }
            if (DO_KV) {
                *reinterpret_cast<uint2*>(kh + off + i0) = o2;
                *reinterpret_cast<uint2*>(kh + off + HALF + i0) = o3;
            }
            if (HAS_VE && DO_KV) {
                *reinterpret_cast<uint2*>(vp + off + i0) = o4;
                *reinterpret_cast<uint2*>(vp + off + HALF + i0) = o5;
            }
        }
        const uint32_t fw = valid ? (mq | (mk << 4) | (mv << 8)) : 0u;
        if (fw != 0u) {
            const int slot = atomicAdd(&s_nfix, 1);
            if (slot < kFixPerBlock) {
                FixItem item;
                item.chunk_lo = (uint32_t)tid;
                item.code = fw | ((uint32_t)(tid >> 32) << 16);
                item.pad0 = item.pad1 = 0u;
                item.rq = rq;
                item.rk = rk;
                s_fix[slot] = item;
            }
        }
    }
    // The repairs: after the barrier every fast-path store of the block is ordered before them.
    __syncthreads();
    const int nf = s_nfix;
    if (nf == 0) return;
    const FixParams fp{q, k, v, ve, gate, qh, kh, vp, tab64, T, H, eps};
    if (nf <= kFixPerBlock) {
        for (int i = threadIdx.x; i < nf; i += blockDim.x) {
            const FixItem item = s_fix[i];
            prologue_fix_chunk<D>((long long)item.chunk_lo | ((long long)(item.code >> 16) << 32), item.code & 0xffffu,
                                  fp, item.rq, item.rk, true);
        }
    } else {
        constexpr uint32_t all = ((PARTS & 1) ? 0x000fu : 0u) | ((PARTS & 2) ? 0x00f0u : 0u) |
                                 ((PARTS & 2) && HAS_VE ? 0xff00u : 0u);
        for (long long it = 0; it < n_iter; ++it) {
            const long long tid = gtid + it * stride;
            if (tid < (long long)n_rows * TPR) prologue_fix_chunk<D>(tid, all, fp, 0.0, 0.0, false);
        }
    }
}

}  // namespace swa
