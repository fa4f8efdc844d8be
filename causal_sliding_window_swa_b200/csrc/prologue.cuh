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
// bound; a pair whose fp32 result could round differently from the exact one is recomputed in
// fp64 (a fraction of a percent of them).
//   norm: r = 1 / sqrt(ss / D + eps) from the sum of squares of the raw inputs (the rotation
//     preserves it) in fp64, where each square and the sum are exact; the inverse square root by
//     two Newton-Raphson steps from the hardware estimate, then rounded once to fp32.
//   rotation: cos and sin are stored as two pieces with 16-bit significands (remainder below
//     2^-33), so every product a * piece is exact in fp32 for a bf16 input a; x = ra * r is then
//     within 4 of its own ulps of the exact value whenever |x| >= 2^-8 r (|a| + |b|).  The test
//     window is 8 ulps, and smaller |x| (partial cancellation) always take the fp64 path.
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
// (g_hi, g_lo) = (fp32(g), fp32(g - g_hi)).  Token bt's 32 gate channels start at
// gate_x + bt * x_stride (32 for the contiguous slice, C for the full layer input).
__global__ void gate_kernel(const __nv_bfloat16* __restrict__ gate_x, const __nv_bfloat16* __restrict__ Wg,
                            float2* __restrict__ gate, int n_rows, int H, FastDiv divH, int x_stride) {
    for (int row = blockIdx.x * blockDim.x + threadIdx.x; row < n_rows; row += gridDim.x * blockDim.x) {
        const int bt = fdiv(row, divH);
        const int h = row - bt * H;
        const __nv_bfloat16* xr = gate_x + (long long)bt * x_stride;
        double z = 0.0;
#pragma unroll 8
        for (int c = 0; c < 32; ++c)
            z = fma((double)__bfloat162float(xr[c]), (double)__bfloat162float(Wg[c * H + h]), z);
        const double g = 2.0 / (1.0 + exp(-z));
        const float g_hi = (float)g;
        gate[row] = make_float2(g_hi, (float)(g - (double)g_hi));
    }
}

// RoPE tables, one entry per (t, i):
//   tab32[t*D/2 + i] = (c_hi, c_lo, s_hi, s_lo) fp32, each piece with a 16-bit significand;
//   tab64[t*D/2 + i] = (cos, sin) fp64, read only by the fp64 path.
__device__ __forceinline__ float round_sig16(double x) {
    // nearest float with at most 16 significant bits (8 low mantissa bits cleared)
    const float f = (float)x;
    const uint32_t u = __float_as_uint(f);
    return __uint_as_float((u + 0x80u) & 0xffffff00u);
}

__global__ void rope_table_kernel(float4* __restrict__ tab32, double2* __restrict__ tab64, int T,
                                  int D, double base) {
    const int half = D / 2;
    const long long n = (long long)T * half;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(idx / half);
        const int i = (int)(idx % half);
        const double theta = pow(base, -2.0 * (double)i / (double)D);
        double s, c;
        sincos((double)t * theta, &s, &c);
        const float c_hi = round_sig16(c), s_hi = round_sig16(s);
        const float c_lo = round_sig16(c - (double)c_hi), s_lo = round_sig16(s - (double)s_hi);
        tab32[idx] = make_float4(c_hi, c_lo, s_hi, s_lo);
        tab64[idx] = make_double2(c, s);
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

// Two rotation pairs (A0, B0), (A1, B1) of one row, scaled by r (r64 in fp64): the bf16 words
// (a'_0, a'_1) and (b'_0, b'_1), each element the correctly rounded bf16 of its exact value.
// w0, w1 = (c_hi, c_lo, s_hi, s_lo) of the two pairs; t64 their fp64 (cos, sin), read only by the
// rare fp64 path.
__device__ __forceinline__ void rope_2pairs_exact(float A0, float B0, float A1, float B1, const float4& w0,
                                                  const float4& w1, const double2* __restrict__ t64, float r,
                                                  double r64, uint32_t& wa, uint32_t& wb) {
    const float A[2] = {A0, A1}, Bv[2] = {B0, B1};
    const float4 w[2] = {w0, w1};
    float xa[2], xb[2];
    bool slow = false;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        // products with a 16-bit piece are exact; one rounding per fma, one per add
        const float ra = fmaf(A[u], w[u].x, -(Bv[u] * w[u].z)) + fmaf(A[u], w[u].y, -(Bv[u] * w[u].w));
        const float rb = fmaf(A[u], w[u].z, Bv[u] * w[u].x) + fmaf(A[u], w[u].w, Bv[u] * w[u].y);
        xa[u] = ra * r;
        xb[u] = rb * r;
        const float small = r * (fabsf(A[u]) + fabsf(Bv[u])) * 0x1p-8f;
        slow |= near_midpoint_8ulp(xa[u]) | near_midpoint_8ulp(xb[u]) | (fabsf(xa[u]) < small) |
                (fabsf(xb[u]) < small);
    }
    wa = pack_bf16x2(xa[0], xa[1]);
    wb = pack_bf16x2(xb[0], xb[1]);
    if (slow) {
        // Rare: these two pairs in fp64, rounded once.
        uint16_t oa[2], ob[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const double2 tw = t64[u];
            const double Ad = (double)A[u], Bd = (double)Bv[u];
            oa[u] = bf16_rn_bits((Ad * tw.x - Bd * tw.y) * r64);
            ob[u] = bf16_rn_bits((Ad * tw.y + Bd * tw.x) * r64);
        }
        wa = oa[0] | ((uint32_t)oa[1] << 16);
        wb = ob[0] | ((uint32_t)ob[1] << 16);
    }
}

// One group of D/8 consecutive threads handles one (b, t, h) row.  Thread c of the group owns
// pairs i in [4c, 4c+4): elements i (in `lo_raw`) and i + D/2 (in `hi_raw`).
template <int D>
__device__ __forceinline__ void rope_rms_pairs4(const uint2& lo_raw, const uint2& hi_raw,
                                                const float4 (&cs)[4],
                                                const double2* __restrict__ tab64, double eps,
                                                uint2& out_lo, uint2& out_hi) {
    constexpr int TPR = D / 8;
    float a[4], b[4];
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
    const double r64 = rsqrt_newton(ss * (1.0 / (double)D) + eps);
    const float r = (float)r64;
    uint32_t wa[2], wb[2];
#pragma unroll
    for (int e = 0; e < 4; e += 2)
        rope_2pairs_exact(a[e], b[e], a[e + 1], b[e + 1], cs[e], cs[e + 1], tab64 + e, r, r64, wa[e >> 1], wb[e >> 1]);
    out_lo = make_uint2(wa[0], wa[1]);
    out_hi = make_uint2(wb[0], wb[1]);
}

// v' = v + g ve for 4 elements: (v + g_hi ve) + g_lo ve in fp32 (two roundings, within 1 ulp
// unless |v'| < 2^-16 |g ve|); fp64 when that could cross a bf16 rounding midpoint.
__device__ __forceinline__ uint2 gated_add4(const uint2& vw, const uint2& ew, float g_hi, float g_lo,
                                            double g64) {
    float v[4], e4[4];
    unpack4(vw, v);
    unpack4(ew, e4);
    uint32_t w[2];
    bool slow = false;
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
        float x[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            x[u] = fmaf(g_lo, e4[e + u], fmaf(g_hi, e4[e + u], v[e + u]));
            slow |= near_midpoint_8ulp(x[u]) | (fabsf(x[u]) < fabsf(g_hi * e4[e + u]) * 0x1p-16f);
        }
        w[e >> 1] = pack_bf16x2(x[0], x[1]);
    }
    if (slow) {
#pragma unroll
        for (int e = 0; e < 4; e += 2)
            w[e >> 1] = (uint32_t)bf16_rn_bits(fma(g64, (double)e4[e], (double)v[e])) |
                        ((uint32_t)bf16_rn_bits(fma(g64, (double)e4[e + 1], (double)v[e + 1])) << 16);
    }
    return make_uint2(w[0], w[1]);
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
    const long long gtid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
    // Every thread of a warp runs the same number of iterations, so the shuffles always see the
    // full warp; rows past the end are computed on zeros and not stored.
    const long long n_iter = ((long long)n_rows * TPR + stride - 1) / stride;
    // The attention kernel that follows takes its work items from this counter.
    if (gtid == 0) {
        sched[0] = 0;
        sched[1] = 0;
    }
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
        constexpr bool DO_Q = (PARTS & 1) != 0, DO_KV = (PARTS & 2) != 0;
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
        const double2* t64 = tab64 + (long long)t * HALF + i0;
        uint2 o0, o1, o2, o3;
        if (DO_Q) rope_rms_pairs4<D>(raw[0], raw[1], cs, t64, eps, o0, o1);
        if (DO_KV) rope_rms_pairs4<D>(raw[2], raw[3], cs, t64, eps, o2, o3);
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
                const double g64 = (double)gw.x + (double)gw.y;
                *reinterpret_cast<uint2*>(vp + off + i0) = gated_add4(raw[4], raw[6], gw.x, gw.y, g64);
                *reinterpret_cast<uint2*>(vp + off + HALF + i0) = gated_add4(raw[5], raw[7], gw.x, gw.y, g64);
            }
        }
    }
}

}  // namespace swa
