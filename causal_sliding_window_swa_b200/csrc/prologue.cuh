// prologue.cuh -- the HBM-bound steps before the attention product:
//   * RoPE on q and k, then parameter-free RMS normalisation (intelliparadigm "GPT-2 for $73",
//     section 2.2: q, k = norm(rope(q)), norm(rope(k)); section 2.1: RMSNorm without gamma/beta);
//   * the gated value embedding v' = v + 2 sigmoid(x[..., :32] . Wg[:, h]) * ve (PaperWeekly
//     repost, "Value Embeddings" paragraph), one gate per (b, t, h).
// Pair layout of the rotation: (i, i + D/2), theta_i = base^(-2i/D), position t rotates
// (a, b) -> (a cos - b sin, a sin + b cos).
//
// Rounding.  Every output element is the correctly rounded bf16 (nearest, ties to even) of the
// exact value of its definition.  The common path runs in fp32 with a rigorous bound E on its
// error; an element whose fp32 value lies within E of a bf16 rounding midpoint (about 1e-4 of
// them) is recomputed in fp64.  So the tensor-core operands do not depend on how the arithmetic
// was organised (an fp32-only pipeline flips the last bf16 bit of ~1e-4 of the elements, which
// moves single attention scores by ~1e-3).
//   rotation: cos and sin are stored as two 16-bit-significand pieces (hi + lo, remainder below
//     2^-33), so a * hi and a * lo are exact in fp32 for a bf16 input a; ra = (a c_hi - b s_hi)
//     + (a c_lo - b s_lo) carries an error of at most 2^-23 |ra| + 2^-32 (|a| + |b|).
//   norm: the sum of squares is taken over the raw inputs (the rotation preserves it) in fp64,
//     where each square is exact; r = 1 / sqrt(ss / D + eps) in fp64, rounded once to fp32.
//   gate: the 32-term dot product and 2 sigmoid(z) in fp64, rounded once to fp32.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace swa {

// RoPE tables, one entry per (t, i):
//   tab32[t*D/2 + i] = (c_hi, c_lo, s_hi, s_lo) fp32, each piece with a 16-bit significand;
//   tab64[t*D/2 + i] = (cos, sin) fp64, read only when an element falls back to fp64.
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

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint16_t bf16_rn_bits(double x) {
    return __bfloat16_as_ushort(__double2bfloat16(x));
}

__device__ __forceinline__ uint4 pack8_bits(const uint16_t (&o)[8]) {
    uint4 r;
    r.x = o[0] | ((uint32_t)o[1] << 16);
    r.y = o[2] | ((uint32_t)o[3] << 16);
    r.z = o[4] | ((uint32_t)o[5] << 16);
    r.w = o[6] | ((uint32_t)o[7] << 16);
    return r;
}

// True if |x - m| <= E for the bf16 rounding midpoint m just above |x|'s bf16 truncation: the
// only midpoint within reach of an error much smaller than half a bf16 ulp.
__device__ __forceinline__ bool near_bf16_midpoint(float x, float E) {
    const float m = __uint_as_float((__float_as_uint(x) & 0xffff0000u) | 0x8000u);
    return fabsf(x - m) <= E;
}

// One group of D/16 consecutive threads handles one (b, t, h) row of D elements.  Thread c of
// the group owns elements [8c, 8c+8) and their rotation partners [8c + D/2, 8c + D/2 + 8):
// two 16-byte loads per tensor; the sum of squares is reduced over the group with shuffles.
template <int D>
__device__ __forceinline__ void rope_rms_row(const __nv_bfloat16* __restrict__ src,
                                             __nv_bfloat16* __restrict__ dst, long long off,
                                             int i0, const float4 (&cs)[8],
                                             const double2* __restrict__ tab64_row, double eps,
                                             bool valid) {
    constexpr int HALF = D / 2;
    constexpr int TPR = D / 16;
    float a[8], b[8];
    if (valid) {
        unpack8(ldg_stream(src + off + i0), a);
        unpack8(ldg_stream(src + off + HALF + i0), b);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = b[e] = 0.f;
    }
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const double ad = (double)a[e], bd = (double)b[e];
        ss = fma(ad, ad, ss);
        ss = fma(bd, bd, ss);
    }
#pragma unroll
    for (int m = TPR / 2; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const double r64 = 1.0 / sqrt(ss / (double)D + eps);
    const float r = (float)r64;

    uint16_t oa[8], ob[8];
    bool slow = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4 w = cs[e];   // (c_hi, c_lo, s_hi, s_lo)
        const float ra = fmaf(a[e], w.x, -(b[e] * w.z)) + fmaf(a[e], w.y, -(b[e] * w.w));
        const float rb = fmaf(a[e], w.z, b[e] * w.x) + fmaf(a[e], w.w, b[e] * w.y);
        const float xa = ra * r, xb = rb * r;
        const float K = r * (fabsf(a[e]) + fabsf(b[e])) * 0x1p-31f;
        slow |= near_bf16_midpoint(xa, fmaf(fabsf(xa), 0x1p-21f, K));
        slow |= near_bf16_midpoint(xb, fmaf(fabsf(xb), 0x1p-21f, K));
        oa[e] = bf16_rn_bits(xa);
        ob[e] = bf16_rn_bits(xb);
    }
    if (slow) {
        // Rare: recompute this thread's elements in fp64 and round once.
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double2 w = tab64_row[i0 + e];
            const double ad = (double)a[e], bd = (double)b[e];
            oa[e] = bf16_rn_bits((ad * w.x - bd * w.y) * r64);
            ob[e] = bf16_rn_bits((ad * w.y + bd * w.x) * r64);
        }
    }
    if (valid) {
        *reinterpret_cast<uint4*>(dst + off + i0) = pack8_bits(oa);
        *reinterpret_cast<uint4*>(dst + off + HALF + i0) = pack8_bits(ob);
    }
}

// v' = v + g ve for 8 elements: fp32 fma with error at most 2^-23 (|g ve| + |v'|); fp64 when
// close to a bf16 rounding midpoint.
__device__ __forceinline__ uint4 gated_add8(const uint4& vw, const uint4& ew, float gf, double g64) {
    float v[8], e8[8];
    unpack8(vw, v);
    unpack8(ew, e8);
    uint16_t o[8];
    bool slow = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float x = fmaf(gf, e8[e], v[e]);
        slow |= near_bf16_midpoint(x, (fabsf(gf * e8[e]) + fabsf(x)) * 0x1p-22f);
        o[e] = bf16_rn_bits(x);
    }
    if (slow) {
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = bf16_rn_bits(fma(g64, (double)e8[e], (double)v[e]));
    }
    return pack8_bits(o);
}

template <int D, bool HAS_VE>
__global__ void __launch_bounds__(256) prologue_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ ve,
    const __nv_bfloat16* __restrict__ gate_x, const __nv_bfloat16* __restrict__ Wg,
    __nv_bfloat16* __restrict__ qh, __nv_bfloat16* __restrict__ kh, __nv_bfloat16* __restrict__ vp,
    const float4* __restrict__ tab32, const double2* __restrict__ tab64, long long n_rows, int T,
    int H, double eps) {
    constexpr int TPR = D / 16;          // threads per row (8 or 4); divides 32
    constexpr int HALF = D / 2;
    constexpr int GCH = 32 / TPR;        // gate channels per thread
    const long long gtid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
    // Every thread of a warp runs the same number of iterations, so the shuffles below always
    // see the full warp; rows past the end are computed on zeros and not stored.
    const long long n_iter = (n_rows * TPR + stride - 1) / stride;
    for (long long it = 0; it < n_iter; ++it) {
        const long long tid = gtid + it * stride;
        const long long row = tid / TPR;          // (b*T + t)*H + h
        const int c = (int)(tid % TPR);
        const bool valid = row < n_rows;
        const long long rr = valid ? row : 0;
        const int h = (int)(rr % H);
        const long long bt = rr / H;
        const int t = (int)(bt % T);
        const int i0 = 8 * c;
        const long long off = rr * D;

        float4 cs[8];
        {
            const float4* tp = tab32 + (long long)t * HALF + i0;
#pragma unroll
            for (int e = 0; e < 8; ++e) cs[e] = __ldg(tp + e);
        }
        const double2* t64 = tab64 + (long long)t * HALF;
        rope_rms_row<D>(q, qh, off, i0, cs, t64, eps, valid);
        rope_rms_row<D>(k, kh, off, i0, cs, t64, eps, valid);

        if constexpr (HAS_VE) {
            double z = 0.0;
            if (valid) {
                const __nv_bfloat16* xr = gate_x + bt * 32 + c * GCH;
#pragma unroll
                for (int e = 0; e < GCH; ++e)
                    z = fma((double)__bfloat162float(xr[e]),
                            (double)__bfloat162float(Wg[(c * GCH + e) * H + h]), z);
            }
#pragma unroll
            for (int m = TPR / 2; m >= 1; m >>= 1) z += __shfl_xor_sync(0xffffffffu, z, m);
            const double g64 = 2.0 / (1.0 + exp(-z));
            const float gf = (float)g64;
            if (valid) {
                const uint4 oa = gated_add8(ldg_stream(v + off + i0), ldg_stream(ve + off + i0), gf, g64);
                const uint4 ob = gated_add8(ldg_stream(v + off + HALF + i0),
                                            ldg_stream(ve + off + HALF + i0), gf, g64);
                *reinterpret_cast<uint4*>(vp + off + i0) = oa;
                *reinterpret_cast<uint4*>(vp + off + HALF + i0) = ob;
            }
        }
    }
}

}  // namespace swa
