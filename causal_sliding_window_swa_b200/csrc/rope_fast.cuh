// rope_fast.cuh -- the fp32 prologue of the layer's forward path: RoPE then parameter-free RMS
// normalisation of q and k (intelliparadigm "GPT-2 for $73", section 2.2: q, k = norm(rope(q)),
// norm(rope(k)); section 2.1: RMSNorm without gamma), and the gated value embedding
// v' = v + g ve (PaperWeekly repost, "Value Embeddings" paragraph), all in fp32 with one rounding
// to bf16 at the end.
//
// The same arithmetic runs in two places: inside the attention kernel, on the raw query tile in
// shared memory (so qhat never goes through HBM), and in prologue_fast_kernel below (khat and v'
// for the attention kernel; qhat as well for the backward's recompute).  Both follow the layout
// fixed here, so they produce the same bits:
//   a row of D elements is split into four quarters; quarter c owns the RoPE pairs
//   i in [c QP, c QP + QP), QP = D / 8, i.e. elements a_i = x[i] and b_i = x[i + D/2];
//   ss_c = sum over its pairs, in order, of (a_i^2, b_i^2) accumulated as an fp32 pair, then
//   ss_c = lo + hi;  ss = (ss_0 + ss_1) + (ss_2 + ss_3);  r = rsqrt(ss / D + eps);
//   a' = bf16((a cos - b sin) r), b' = bf16((a sin + b cos) r), cos / sin the fp32 roundings of
//   the fp64 values at angle t base^(-2i/D).
// Error bound: the squares of bf16 inputs are exact in fp32, and every other step rounds once in
// fp32, so each output is the bf16 rounding of a value within a few fp32 ulps of r (|a| + |b|) of
// the exact one; it therefore differs from the correctly rounded bf16 of the exact value by at most
// one bf16 ulp, and only when the exact value lies within that distance of a rounding midpoint
// (about one element in 10^4 on unit-scale data).
//
// v' = bf16(fma(g, ve, v)) with g the fp32 rounding of the gate 2 sigmoid(x[:32] . Wg[:, h]) (the
// gate itself is computed in fp64 by gate_kernel).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace swa {

// Element i (0..7) of 8 packed bf16 in a 16-byte word, as fp32.
__device__ __forceinline__ float bf16_at(const uint4& u, int i) {
    const uint32_t w = (i >> 1) == 0 ? u.x : (i >> 1) == 1 ? u.y : (i >> 1) == 2 ? u.z : u.w;
    return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
}

// Partial sum of squares of one quarter from its packed bf16 words: pair i has a_i (word i / 8 of
// wa) and b_i (word i / 8 of wb); QP = 8 NW pairs, accumulated in order as an fp32 pair.
template <int NW>
__device__ __forceinline__ float quarter_sumsq(const uint4 (&wa)[NW], const uint4 (&wb)[NW]) {
    uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8 * NW; ++i) {
        const uint64_t x = f2_pack(bf16_at(wa[i >> 3], i & 7), bf16_at(wb[i >> 3], i & 7));
        acc = f2_fma(x, x, acc);
    }
    float lo, hi;
    f2_unpack(acc, lo, hi);
    return lo + hi;
}

// The row's scale from the four quarters' partial sums.
__device__ __forceinline__ float rms_scale4(float s0, float s1, float s2, float s3, float inv_d, float eps) {
    const float ss = (s0 + s1) + (s2 + s3);
    return rsqrtf(fmaf(ss, inv_d, eps));
}

// One rotated, scaled pair -> two bf16 (round to nearest even).
__device__ __forceinline__ void rope_pair(float a, float b, float c, float s, float r, float& oa, float& ob) {
    oa = __fmul_rn(fmaf(a, c, -__fmul_rn(b, s)), r);
    ob = __fmul_rn(fmaf(a, s, __fmul_rn(b, c)), r);
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// 8 bf16 (one 16-byte word) -> 8 fp32.
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// fp32 RoPE table: tabf[t * D/2 + i] = (cos, sin) of t base^(-2i/D), rounded from fp64.
__device__ __forceinline__ float2 rope_cs(const float2* __restrict__ tabf, int t, int half, int i) {
    return __ldg(tabf + (long long)t * half + i);
}

// Rotate + scale the 8 NW pairs of one quarter, packed bf16 in and out: words e of wa / wb hold
// a_{8e..8e+7} / b_{8e..8e+7}; cs[p] = (cos, sin) of pairs 2p and 2p + 1.
template <int NW>
__device__ __forceinline__ void rope_quarter(const uint4 (&wa)[NW], const uint4 (&wb)[NW], const float4 (&cs)[4 * NW],
                                             float r, uint4 (&oa)[NW], uint4 (&ob)[NW]) {
#pragma unroll
    for (int e = 0; e < NW; ++e) {
        uint32_t xa[4], xb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float4 c = cs[4 * e + u];
            float a0, b0, a1, b1;
            rope_pair(bf16_at(wa[e], 2 * u), bf16_at(wb[e], 2 * u), c.x, c.y, r, a0, b0);
            rope_pair(bf16_at(wa[e], 2 * u + 1), bf16_at(wb[e], 2 * u + 1), c.z, c.w, r, a1, b1);
            xa[u] = bf16x2_rn(a0, a1);
            xb[u] = bf16x2_rn(b0, b1);
        }
        oa[e] = make_uint4(xa[0], xa[1], xa[2], xa[3]);
        ob[e] = make_uint4(xb[0], xb[1], xb[2], xb[3]);
    }
}

// Elementwise v' = bf16(fma(g, ve, v)) of 8 elements.
__device__ __forceinline__ uint4 gated_add8_fast(const uint4& vw, const uint4& ew, float g) {
    float v[8], e[8];
    unpack8(vw, v);
    unpack8(ew, e);
    return make_uint4(bf16x2_rn(fmaf(g, e[0], v[0]), fmaf(g, e[1], v[1])),
                      bf16x2_rn(fmaf(g, e[2], v[2]), fmaf(g, e[3], v[3])),
                      bf16x2_rn(fmaf(g, e[4], v[4]), fmaf(g, e[5], v[5])),
                      bf16x2_rn(fmaf(g, e[6], v[6]), fmaf(g, e[7], v[7])));
}

// The fp32 prologue over rows in HBM.  Blocks [0, nb_q) take query rows (B T H of them; qhat),
// blocks [nb_q, nb_q + nb_k) key rows (B T Hkv; khat), the rest value rows (v' = v + g ve on
// value-embedding layers).  Query / key blocks: four consecutive threads per row, thread c the
// row's quarter c (the layout of the arithmetic above; the four partial sums meet by shuffles).
// Value blocks: each thread 32 consecutive elements of one row (D / 32 threads per row).
// Rows are (b, t, head) in the (B, T, heads, D) layout; t = (row / heads) mod T.
struct FastProParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const __nv_bfloat16* ve;
    const float2* gate;       // (B T Hkv) (g_hi, g_lo); g = g_hi is used
    __nv_bfloat16* qh;
    __nv_bfloat16* kh;
    __nv_bfloat16* vp;
    const float2* tabf;
    int n_q, n_k, n_v;        // rows of each part
    int nb_q, nb_k;           // blocks of the q and k parts
    int H, Hkv, T;
    float inv_d, eps;
    int* sched;               // the attention kernel's counters, zeroed here (or null)
};

template <int D, bool HAS_VE>
__global__ void __launch_bounds__(256) prologue_fast_kernel(const FastProParams p) {
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
        float4 cs[QP / 2];
        const float4* tp = reinterpret_cast<const float4*>(p.tabf + (long long)t * HALF + c * QP);
#pragma unroll
        for (int e = 0; e < NW; ++e) {
            wa[e] = live ? ldg_stream16(xr + c * QP + 8 * e) : make_uint4(0u, 0u, 0u, 0u);
            wb[e] = live ? ldg_stream16(xr + HALF + c * QP + 8 * e) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int e = 0; e < QP / 2; ++e) cs[e] = __ldg(tp + e);
        const float part = quarter_sumsq<NW>(wa, wb);
        const int lane = threadIdx.x & 31;
        const int base = lane & ~3;
        const float s0 = __shfl_sync(0xffffffffu, part, base + 0);
        const float s1 = __shfl_sync(0xffffffffu, part, base + 1);
        const float s2 = __shfl_sync(0xffffffffu, part, base + 2);
        const float s3 = __shfl_sync(0xffffffffu, part, base + 3);
        const float r = rms_scale4(s0, s1, s2, s3, p.inv_d, p.eps);
        uint4 oa[NW], ob[NW];
        rope_quarter<NW>(wa, wb, cs, r, oa, ob);
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
        const __nv_bfloat16* vr = p.v + e0;
        uint4 vw[4], ew[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) vw[e] = ldg_stream16(vr + 8 * e);
        float g = 0.f;
        if constexpr (HAS_VE) {
#pragma unroll
            for (int e = 0; e < 4; ++e) ew[e] = ldg_stream16(p.ve + e0 + 8 * e);
            g = __ldg(p.gate + row).x;
        }
        uint4* dr = reinterpret_cast<uint4*>(p.vp + e0);
#pragma unroll
        for (int e = 0; e < 4; ++e) dr[e] = HAS_VE ? gated_add8_fast(vw[e], ew[e], g) : vw[e];
    }
}

}  // namespace swa
