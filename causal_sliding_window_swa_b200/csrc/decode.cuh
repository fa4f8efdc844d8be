// decode.cuh -- one generation step with a key/value cache: the new token at position `pos` of
// every sequence goes through the layer's prologue (RoPE, RMS QK-norm, gated value embedding;
// intelliparadigm "GPT-2 for $73", sections 2.1, 2.2 and the "Value Embeddings" paragraph of
// the PaperWeekly repost), its k-hat and v' are appended to the caches, and its query attends
// to the cached keys inside its window ("Let's reproduce GPT-2 (124M)" notes, section 19, which
// lists a KV cache among the missing pieces):
//   out[b,h,:] = sum_{j in J} softmax_j(qhat . khat_j / sqrt(D)) v'_j,  J = [max(0, pos-W+1), pos].
//
// The per-element arithmetic of the prologue is the prefill path's (prologue.cuh), so the cache
// entries are bit-identical to the k-hat / v' the prefill path writes for the same token.
// Attention: the window's keys are cut into chunks of CK keys, one CTA per (chunk, b, h).  The
// softmax offset is fixed at M0 = sqrt(D) (1 + 2^-6) (the QK-norm bound used by the prefill
// kernel), so chunk results need no rescaling: each chunk writes sum_j p_j v'_j and sum_j p_j,
// and a third kernel adds the chunks in order (deterministic) and divides.  Scores, exponentials
// and the weighted sums are fp32; nothing goes through bf16 except the final output.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "prologue.cuh"
#include "ptx.cuh"

namespace swa {

constexpr int kDecodeChunk = 128;        // fewest keys per CTA of the attention kernel (the host picks
                                         // a multiple of 32 from here up to fill the GPU's CTA slots)

// Prologue of the new token: rows r = b*H + h (H = the head count of this pass); D/8 threads per
// row as in the prefill prologue.  PARTS: bit 0 qhat (to the workspace), bit 1 khat and v' (to the
// caches); grouped-query layers run the query rows and the key/value rows as two passes.
// The block first builds the RoPE row of position `pos` in shared memory, with the same split as
// the prefill table (16-bit-significand pieces and the fp64 pair for the fallback).  On
// value-embedding layers the first thread of each row computes the gate 2 sigmoid(x . Wg[:, h]) in
// fp64 in the order of the prefill gate kernel, so the value is the same.
template <int D, bool HAS_VE, int PARTS = 3>
__global__ void __launch_bounds__(256) decode_prologue_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ ve,
    const __nv_bfloat16* __restrict__ gate_x, const __nv_bfloat16* __restrict__ Wg,
    __nv_bfloat16* __restrict__ qh, __nv_bfloat16* __restrict__ k_cache,
    __nv_bfloat16* __restrict__ v_cache, int n_rows, int H, int Tmax, int pos, double base,
    double eps) {
    constexpr int TPR = D / 8;
    constexpr int HALF = D / 2;
    __shared__ float4 s_tab32[HALF];
    __shared__ double2 s_tab64[HALF];
    for (int i = threadIdx.x; i < HALF; i += blockDim.x) {
        const double theta = pow(base, -2.0 * (double)i / (double)D);
        double sn, cs;
        sincos((double)pos * theta, &sn, &cs);
        float c_hi, c_lo, s_hi, s_lo;
        rope_split(cs, c_hi, c_lo);
        rope_split(sn, s_hi, s_lo);
        s_tab32[i] = make_float4(c_hi, c_lo, s_hi, s_lo);
        s_tab64[i] = make_double2(cs, sn);
    }
    __syncthreads();
    const int rows_per_block = blockDim.x / TPR;
    const int c = threadIdx.x % TPR;
    const int i0 = 4 * c;
    // Every thread of a warp runs the same number of iterations (rows past the end compute on
    // zeros and store nothing), so the shuffles inside the row functions see the whole warp.
    for (int row0 = blockIdx.x * rows_per_block; row0 < n_rows; row0 += gridDim.x * rows_per_block) {
        const int row_raw = row0 + (int)threadIdx.x / TPR;
        const bool valid = row_raw < n_rows;
        const int row = valid ? row_raw : 0;
        const int b = row / H;
        const int h = row - b * H;
        const long long in_off = (long long)row * D;
        const long long cache_off = (((long long)b * Tmax + pos) * H + h) * D;
        constexpr bool DO_Q = (PARTS & 1) != 0, DO_KV = (PARTS & 2) != 0;
        uint2 raw[8];
        float2 gw = make_float2(0.f, 0.f);
        if (HAS_VE && DO_KV) {
            // gate of this row by its first thread, then shared with the row's other threads
            if (c == 0 && valid) {
                const __nv_bfloat16* xr = gate_x + (long long)b * 32;
                double z = 0.0;
                for (int cc = 0; cc < 32; ++cc)
                    z = fma((double)__bfloat162float(xr[cc]), (double)__bfloat162float(Wg[cc * H + h]), z);
                const double g = 2.0 / (1.0 + exp(-z));
                gw.x = (float)g;
                gw.y = (float)(g - (double)gw.x);
            }
            const int src = ((int)(threadIdx.x & 31u) / TPR) * TPR;
            gw.x = __shfl_sync(0xffffffffu, gw.x, src);
            gw.y = __shfl_sync(0xffffffffu, gw.y, src);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) raw[e] = make_uint2(0u, 0u);
        if (valid) {
            if (DO_Q) {
                raw[0] = ldg_stream8(q + in_off + i0);
                raw[1] = ldg_stream8(q + in_off + HALF + i0);
            }
            if (DO_KV) {
                raw[2] = ldg_stream8(k + in_off + i0);
                raw[3] = ldg_stream8(k + in_off + HALF + i0);
                raw[4] = ldg_stream8(v + in_off + i0);
                raw[5] = ldg_stream8(v + in_off + HALF + i0);
            }
            if (HAS_VE && DO_KV) {
                raw[6] = ldg_stream8(ve + in_off + i0);
                raw[7] = ldg_stream8(ve + in_off + HALF + i0);
            }
        }
        float4 cs4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) cs4[e] = s_tab32[i0 + e];
        uint2 o0, o1, o2, o3;
        if (DO_Q) rope_rms_exact4<D>(raw[0], raw[1], cs4, s_tab64 + i0, eps, o0, o1);
        if (DO_KV) rope_rms_exact4<D>(raw[2], raw[3], cs4, s_tab64 + i0, eps, o2, o3);
        if (valid && DO_Q) {
            *reinterpret_cast<uint2*>(qh + in_off + i0) = o0;
            *reinterpret_cast<uint2*>(qh + in_off + HALF + i0) = o1;
        }
        if (valid && DO_KV) {
            *reinterpret_cast<uint2*>(k_cache + cache_off + i0) = o2;
            *reinterpret_cast<uint2*>(k_cache + cache_off + HALF + i0) = o3;
            if (HAS_VE) {
                const double g64 = (double)gw.x + (double)gw.y;
                *reinterpret_cast<uint2*>(v_cache + cache_off + i0) = gated_add4(raw[4], raw[6], gw.x, gw.y, g64);
                *reinterpret_cast<uint2*>(v_cache + cache_off + HALF + i0) =
                    gated_add4(raw[5], raw[7], gw.x, gw.y, g64);
            } else {
                *reinterpret_cast<uint2*>(v_cache + cache_off + i0) = raw[4];
                *reinterpret_cast<uint2*>(v_cache + cache_off + HALF + i0) = raw[5];
            }
        }
    }
}

// DPL consecutive bf16 features as raw bits: 8 bytes (DPL = 4) or 4 bytes (DPL = 2).
template <int DPL>
struct Raw;
template <>
struct Raw<4> {
    uint2 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = *reinterpret_cast<const uint2*>(p); }
    __device__ __forceinline__ void zero() { u = make_uint2(0u, 0u); }
    __device__ __forceinline__ void unpack(float (&f)[4]) const {
        f[0] = __uint_as_float(u.x << 16);
        f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16);
        f[3] = __uint_as_float(u.y & 0xffff0000u);
    }
};
template <>
struct Raw<2> {
    uint32_t u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = *reinterpret_cast<const uint32_t*>(p); }
    __device__ __forceinline__ void zero() { u = 0u; }
    __device__ __forceinline__ void unpack(float (&f)[2]) const {
        f[0] = __uint_as_float(u << 16);
        f[1] = __uint_as_float(u & 0xffff0000u);
    }
};

// Attention of the new token over one chunk of cached keys.  Grid B*H*n_chunks, 4 warps; the
// lanes of a warp split the D features (D/32 each).  Per iteration the block takes 32 keys, eight
// per warp (keys w, w+4, ..., w+28 of the block): the warp loads their K and V pieces first, then
// reduces the eight dot products together, so sixteen loads per lane are in flight at once.
// Partial results: part[(row * n_chunks + chunk) * (D + 2) + d] = sum_j p_j v'_j[d],
// [.. + D] = sum_j p_j.  With doc_start (one int per sequence: the first position of the new
// token's document; document-boundary mask) the keys before it are skipped: a chunk that lies
// entirely before it writes zeros.
template <int D>
__global__ void __launch_bounds__(128) decode_attn_kernel(
    const __nv_bfloat16* __restrict__ qh, const __nv_bfloat16* __restrict__ k_cache,
    const __nv_bfloat16* __restrict__ v_cache, float* __restrict__ part, int H, int Hkv, int Tmax,
    int lo, int n_keys, int n_chunks, int chunk_keys, float c1, float c2, const int* __restrict__ doc_start) {
    constexpr int DPL = D / 32;          // features per lane
    constexpr int U = 8;                 // keys per warp per iteration
    const int row = (int)(blockIdx.x / (unsigned)n_chunks);    // b*H + h
    const int chunk = (int)(blockIdx.x - (unsigned)row * (unsigned)n_chunks);
    const int b = row / H;
    const int h = row - b * H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ float s_o[4][D];
    __shared__ float s_l[4];
    float qf[DPL];
    {
        Raw<DPL> rq;
        rq.load(qh + (long long)row * D + lane * DPL);
        rq.unpack(qf);
    }
    float o[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[e] = 0.f;
    float l = 0.f;
    // first key of this chunk, past the document start if there is one (key index j is position lo + j)
    const int jmin = doc_start != nullptr ? max(0, min(__ldg(doc_start + b), lo + n_keys - 1) - lo) : 0;
    const int key_begin = max(chunk * chunk_keys, jmin);
    const int key_end = min(chunk * chunk_keys + chunk_keys, n_keys);
    const int hk = h / (H / Hkv);                           // key/value head of this query head
    const long long stride = (long long)Hkv * D;            // between consecutive positions
    const __nv_bfloat16* kbase = k_cache + ((long long)b * Tmax + lo) * stride + (long long)hk * D + lane * DPL;
    const __nv_bfloat16* vbase = v_cache + ((long long)b * Tmax + lo) * stride + (long long)hk * D + lane * DPL;
    for (int j0 = key_begin + warp; j0 < key_end; j0 += 4 * U) {
        Raw<DPL> rk[U], rv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = j0 + 4 * u;
            if (j < key_end) {
                rk[u].load(kbase + (long long)j * stride);
                rv[u].load(vbase + (long long)j * stride);
            } else {
                rk[u].zero();
                rv[u].zero();
            }
        }
        float s[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float kf[DPL];
            rk[u].unpack(kf);
            s[u] = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) s[u] = fmaf(qf[e], kf[e], s[u]);
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
            for (int u = 0; u < U; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], m);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (j0 + 4 * u >= key_end) continue;
            const float p = ex2_approx(fmaf(s[u], c1, -c2));
            l += p;
            float vf[DPL];
            rv[u].unpack(vf);
#pragma unroll
            for (int e = 0; e < DPL; ++e) o[e] = fmaf(p, vf[e], o[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) s_o[warp][lane * DPL + e] = o[e];
    if (lane == 0) s_l[warp] = l;
    __syncthreads();
    float* dst = part + ((long long)row * n_chunks + chunk) * (D + 2);
    for (int d = threadIdx.x; d < D; d += blockDim.x)
        dst[d] = (s_o[0][d] + s_o[1][d]) + (s_o[2][d] + s_o[3][d]);
    if (threadIdx.x == 0) dst[D] = (s_l[0] + s_l[1]) + (s_l[2] + s_l[3]);
}

// Adds the chunks of each row in order and writes out = o / l (bf16) and lse = M0 + ln l.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float* __restrict__ part,
                                                          __nv_bfloat16* __restrict__ out,
                                                          float* __restrict__ lse, int n_chunks,
                                                          float m0) {
    const int row = blockIdx.x;
    const int d = threadIdx.x;
    const float* src = part + (long long)row * n_chunks * (D + 2);
    float o = 0.f, l = 0.f;
    for (int c = 0; c < n_chunks; ++c) {
        o += src[(long long)c * (D + 2) + d];
        l += src[(long long)c * (D + 2) + D];
    }
    out[(long long)row * D + d] = __float2bfloat16_rn(o / l);
    if (d == 0 && lse != nullptr) lse[row] = m0 + logf(l);
}

}  // namespace swa
