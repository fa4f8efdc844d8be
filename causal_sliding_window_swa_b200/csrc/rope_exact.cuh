// rope_exact.cuh -- the prologue of the layer's forward path, exactly rounded: RoPE then
// parameter-free RMS normalisation of q and k (intelliparadigm "GPT-2 for $73", section 2.2:
// q, k = norm(rope(q)), norm(rope(k)); section 2.1: RMSNorm without gamma), and the gated value
// embedding v' = v + g ve (PaperWeekly repost, "Value Embeddings" paragraph).  Every output is
// the bf16 rounding (nearest, ties to even) of an fp64 evaluation of its definition, so it is the
// correctly rounded bf16 of the exact value except when that value lies within about 2^-50 of a
// rounding midpoint (the same values the oracle's parity mode produces).
//
// The same arithmetic runs in two places: inside the attention kernel, on the raw query tile in
// shared memory (so qhat need not go through HBM), and in prologue_exact_kernel below.  Both use
// the layout fixed here, so they produce the same bits:
//   a row of D elements is split into four quarters; quarter c owns the RoPE pairs
//   i in [c QP, c QP + QP), QP = D / 8, i.e. elements a_i = x[i] and b_i = x[i + D/2];
//   ss_c = sum over its pairs, in order, of a_i^2 then b_i^2, in fp64 (the squares of bf16 values
//   are exact in fp64, and so is their sum unless the magnitudes span more than 2^37);
//   ss = (ss_0 + ss_1) + (ss_2 + ss_3);  r = 1 / sqrt(ss / D + eps) (fp64, two Newton steps);
//   a' = bf16(fma(a, cos, -(b sin)) r), b' = bf16(fma(a, sin, b cos) r), cos / sin the fp64 values
//   at angle t base^(-2i/D).
// v' = bf16(fma(g, ve, v)) in fp64, with g = 2 sigmoid(x[:32] . Wg[:, h]) in fp64 (gate_kernel).
// On B200 fp64 arithmetic runs at half the fp32 rate; these are a few fp64 operations per element
// of an HBM-bound pass.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace swa {

// Element i (0..7) of 8 packed bf16 in a 16-byte word, as fp64 (exact).
__device__ __forceinline__ double bf16_at64(const uint4& u, int i) {
    const uint32_t w = (i >> 1) == 0 ? u.x : (i >> 1) == 1 ? u.y : (i >> 1) == 2 ? u.z : u.w;
    return (double)__uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
}

__device__ __forceinline__ uint32_t bf16_bits_rn(double x) {
    return (uint32_t)__bfloat16_as_ushort(__double2bfloat16(x));
}

// Partial sum of squares of one quarter from its packed bf16 words: word e of wa / wb holds
// a_{8e..8e+7} / b_{8e..8e+7}; pairs in order, a_i^2 then b_i^2.
template <int NW>
__device__ __forceinline__ double quarter_sumsq64(const uint4 (&wa)[NW], const uint4 (&wb)[NW]) {
    double acc = 0.0;
#pragma unroll
    for (int i = 0; i < 8 * NW; ++i) {
        const double a = bf16_at64(wa[i >> 3], i & 7), b = bf16_at64(wb[i >> 3], i & 7);
        acc = fma(a, a, acc);
        acc = fma(b, b, acc);
    }
    return acc;
}

// 1 / sqrt(y), y > 0: the hardware fp32 estimate refined by two Newton-Raphson steps for the
// inverse square root, r <- r (3 - y r^2) / 2 (each squares the relative error: ~2^-22 -> 2^-44
// -> below 2^-52).
__device__ __forceinline__ double rsqrt64(double y) {
    double r = (double)rsqrtf((float)y);
    r = r * fma(-0.5 * y, r * r, 1.5);
    r = r * fma(-0.5 * y, r * r, 1.5);
    return r;
}

// The row's scale from the four quarters' partial sums (fixed order).
__device__ __forceinline__ double rms_scale64(double s0, double s1, double s2, double s3, double inv_d, double eps) {
    return rsqrt64(((s0 + s1) + (s2 + s3)) * inv_d + eps);
}

// Rotate + scale the 8 NW pairs of one quarter: packed bf16 in and out (word e of oa / ob holds
// a'_{8e..8e+7} / b'_{8e..8e+7}); cs[i] = (cos, sin) of the quarter's pair i, read from `tab`.
template <int NW>
__device__ __forceinline__ void rope_quarter64(const uint4 (&wa)[NW], const uint4 (&wb)[NW],
                                               const double2* __restrict__ tab, double r,
                                               uint4 (&oa)[NW], uint4 (&ob)[NW]) {
#pragma unroll
    for (int e = 0; e < NW; ++e) {
        uint32_t xa[4], xb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint32_t pa[2], pb[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = 8 * e + 2 * u + h;
                const double2 cs = __ldg(tab + i);
                const double a = bf16_at64(wa[e], 2 * u + h), b = bf16_at64(wb[e], 2 * u + h);
                pa[h] = bf16_bits_rn(fma(a, cs.x, -(b * cs.y)) * r);
                pb[h] = bf16_bits_rn(fma(a, cs.y, b * cs.x) * r);
            }
            xa[u] = pa[0] | (pa[1] << 16);
            xb[u] = pb[0] | (pb[1] << 16);
        }
        oa[e] = make_uint4(xa[0], xa[1], xa[2], xa[3]);
        ob[e] = make_uint4(xb[0], xb[1], xb[2], xb[3]);
    }
}

// Elementwise v' = bf16(fma(g, ve, v)) of 8 elements, in fp64.
__device__ __forceinline__ uint4 gated_add8_64(const uint4& vw, const uint4& ew, double g) {
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t lo = bf16_bits_rn(fma(g, bf16_at64(ew, 2 * u), bf16_at64(vw, 2 * u)));
        const uint32_t hi = bf16_bits_rn(fma(g, bf16_at64(ew, 2 * u + 1), bf16_at64(vw, 2 * u + 1)));
        w[u] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// The prologue over rows in HBM.  Blocks [0, nb_q) take query rows (B T H of them; qhat), blocks
// [nb_q, nb_q + nb_k) key rows (B T Hkv; khat), the rest value rows (v' = v + g ve, value-embedding
// layers).  Query / key blocks: four consecutive threads per row, thread c the row's quarter c (the
// layout of the arithmetic above; the four partial sums meet by shuffles in the fixed order).
// Value blocks: each thread 32 consecutive elements of one row.  Rows are (b, t, head) in the
// (B, T, heads, D) layout; t = (row / heads) mod T.
struct ExactProParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const __nv_bfloat16* ve;
    const float2* gate;       // (B T Hkv) (g_hi, g_lo): g = g_hi + g_lo
    __nv_bfloat16* qh;
    __nv_bfloat16* kh;
    __nv_bfloat16* vp;
    const double2* tab64;     // (cos, sin) per (t, i), fp64
    int n_q, n_k, n_v;        // rows of each part
    int nb_q, nb_k;           // blocks of the q and k parts
    int H, Hkv, T;
    double inv_d, eps;
    int* sched;               // the attention kernel's counters, zeroed here (or null)
};

template <int D, bool HAS_VE>
__global__ void __launch_bounds__(256) prologue_exact_kernel(const ExactProParams p) {
    constexpr int QP = D / 8;             // pairs per quarter
    constexpr int HALF = D / 2;
    constexpr int NW = QP / 8;            // 16-byte words per half-quarter (2 at D = 128, 1 at D = 64)
    if (blockIdx.x == 0 && threadIdx.x == 0 && p.sched != nullptr) {
        p.sched[0] = 0;
        p.sched[1] = 0;
    }
    const int bid = blockIdx.x;
    if (bid < p.nb_q + p.nb_k) {
        const bool is_q = bid < p.nb_q;
        const int lb = is_q ? bid : bid - p.nb_q;
        const int n_rows = is_q ? p.n_q : p.n_k;
        const int heads = is_q ? p.H : p.Hkv;
        const __nv_bfloat16* src = is_q ? p.q : p.k;
        __nv_bfloat16* dst = is_q ? p.qh : p.kh;
        const int row_raw = lb * 64 + (threadIdx.x >> 2);
        const int c = threadIdx.x & 3;
        const bool live = row_raw < n_rows;    // the whole warp takes part in the shuffles
        const int row = live ? row_raw : 0;
        const int t = (row / heads) % p.T;
        const __nv_bfloat16* xr = src + (long long)row * D;
        uint4 wa[NW], wb[NW];
#pragma unroll
        for (int e = 0; e < NW; ++e) {
            wa[e] = live ? ldg_stream16(xr + c * QP + 8 * e) : make_uint4(0u, 0u, 0u, 0u);
            wb[e] = live ? ldg_stream16(xr + HALF + c * QP + 8 * e) : make_uint4(0u, 0u, 0u, 0u);
        }
        const double part = quarter_sumsq64<NW>(wa, wb);
        const int base = threadIdx.x & 28;     // first lane of this row's four
        const double s0 = __shfl_sync(0xffffffffu, part, base + 0);
        const double s1 = __shfl_sync(0xffffffffu, part, base + 1);
        const double s2 = __shfl_sync(0xffffffffu, part, base + 2);
        const double s3 = __shfl_sync(0xffffffffu, part, base + 3);
        const double r = rms_scale64(s0, s1, s2, s3, p.inv_d, p.eps);
        uint4 oa[NW], ob[NW];
        rope_quarter64<NW>(wa, wb, p.tab64 + (long long)t * HALF + c * QP, r, oa, ob);
        if (live) {
            __nv_bfloat16* dr = dst + (long long)row * D;
#pragma unroll
            for (int e = 0; e < NW; ++e) {
                *reinterpret_cast<uint4*>(dr + c * QP + 8 * e) = oa[e];
                *reinterpret_cast<uint4*>(dr + HALF + c * QP + 8 * e) = ob[e];
            }
        }
    } else {
        // value rows: 32 elements per thread
        const long long e0 = ((long long)(bid - p.nb_q - p.nb_k) * 256 + threadIdx.x) * 32;
        if (e0 >= (long long)p.n_v * D) return;
        const int row = (int)(e0 / D);
        uint4 vw[4], ew[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) vw[e] = ldg_stream16(p.v + e0 + 8 * e);
        double g = 0.0;
        if constexpr (HAS_VE) {
#pragma unroll
            for (int e = 0; e < 4; ++e) ew[e] = ldg_stream16(p.ve + e0 + 8 * e);
            const float2 gg = __ldg(p.gate + row);
            g = (double)gg.x + (double)gg.y;
        }
        uint4* dr = reinterpret_cast<uint4*>(p.vp + e0);
#pragma unroll
        for (int e = 0; e < 4; ++e) dr[e] = HAS_VE ? gated_add8_64(vw[e], ew[e], g) : vw[e];
    }
}

}  // namespace swa
