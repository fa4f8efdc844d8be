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
// Attention: the window's keys are cut into chunks, one CTA per (chunk, b, h) and the chunks of a
// row forming a thread-block cluster.  The softmax offset is fixed at M0 = sqrt(D) (1 + 2^-6) (the
// QK-norm bound used by the prefill kernel), so chunk results need no rescaling: each chunk keeps
// sum_j p_j v'_j and sum_j p_j, and the first CTA of the cluster adds the chunks in order
// (deterministic) and divides.  Scores, exponentials and the weighted sums are fp32; nothing goes
// through bf16 except the final output.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "prologue.cuh"
#include "ptx.cuh"

namespace swa {

// Prologue of the new token: rows r = b*H + h (H = the head count of this pass); D/8 threads per
// row as in the prefill prologue.  PARTS: bit 0 qhat (to the workspace), bit 1 khat and v' (to the
// caches); grouped-query layers run the query rows and the key/value rows as two passes.
// The block first builds the RoPE row of position `pos` in shared memory, with the same split as
// the prefill table (16-bit-significand pieces and the fp64 pair for the fallback).  Meanwhile,
// on value-embedding layers, one thread per row computes the gate 2 sigmoid(x . Wg[:, h]) in fp64
// in the order of the prefill gate kernel, so the value is the same.
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
    // the attention kernel may start now: it streams the cached keys while this kernel runs
    grid_dependents_launch();
    __shared__ float4 s_tab32[HALF];
    __shared__ double2 s_tab64[HALF];
    __shared__ float2 s_gate[32];
    const int rows_per_block = blockDim.x / TPR;      // 16 or 32
    // gate 2 sigmoid(x . Wg[:, h]) of row r in fp64, summed over the 32 channels in order (the
    // prefill gate kernel's order); every load issued before the products
    auto gate_of = [&](int r) -> float2 {
        const int b = r / H, h = r - (r / H) * H;
        const __nv_bfloat16* xr = gate_x + (long long)b * 32;
        float xv[32], wv[32];
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
            xv[cc] = __bfloat162float(xr[cc]);
            wv[cc] = __bfloat162float(Wg[cc * H + h]);
        }
        double z = 0.0;
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) z = fma((double)xv[cc], (double)wv[cc], z);
        const double g = 2.0 / (1.0 + exp(-z));
        const float g_hi = (float)g;
        return make_float2(g_hi, (float)(g - (double)g_hi));
    };
    // The RoPE row of `pos` (threads 32 .. 32 + D/2 - 1) and, at the same time, the gates of the
    // block's first rows (threads 0 .. rows_per_block - 1).
    if (threadIdx.x >= 32 && threadIdx.x < 32 + HALF) {
        const int i = (int)threadIdx.x - 32;
        const double theta = pow(base, -2.0 * (double)i / (double)D);
        double sn, cs;
        sincos((double)pos * theta, &sn, &cs);
        float c_hi, c_lo, s_hi, s_lo;
        rope_split(cs, c_hi, c_lo);
        rope_split(sn, s_hi, s_lo);
        s_tab32[i] = make_float4(c_hi, c_lo, s_hi, s_lo);
        s_tab64[i] = make_double2(cs, sn);
    }
    if (HAS_VE && (PARTS & 2) != 0 && (int)threadIdx.x < rows_per_block) {
        const int r = (int)blockIdx.x * rows_per_block + (int)threadIdx.x;
        if (r < n_rows) s_gate[threadIdx.x] = gate_of(r);
    }
    __syncthreads();
    const int c = threadIdx.x % TPR;
    const int i0 = 4 * c;
    // Every thread of a warp runs the same number of iterations (rows past the end compute on
    // zeros and store nothing), so the shuffles inside the row functions see the whole warp.
    for (int row0 = blockIdx.x * rows_per_block; row0 < n_rows; row0 += gridDim.x * rows_per_block) {
        if (HAS_VE && (PARTS & 2) != 0 && row0 != (int)blockIdx.x * rows_per_block) {
            // later row groups of this block (more rows than the grid covers at once)
            __syncthreads();
            if ((int)threadIdx.x < rows_per_block && row0 + (int)threadIdx.x < n_rows)
                s_gate[threadIdx.x] = gate_of(row0 + (int)threadIdx.x);
            __syncthreads();
        }
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
        if (HAS_VE && DO_KV && valid) gw = s_gate[threadIdx.x / TPR];
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

// ------------------------------------------------------------------- attention of the new token
//
// One CTA per (row b*H + h, chunk of the window), the chunks of a row forming one thread-block
// cluster, launched so that it may start while the token prologue runs: it forms qhat itself and
// waits for that kernel only before it loads the tile with the new token.  A producer warp streams the chunk's K and V' tiles (KB keys x D, 8 KB each) from the
// caches into a four-stage shared-memory ring with TMA; four consumer warps take KB / 4 keys of
// each tile.  Lane l holds features [l DPL, (l + 1) DPL) of qhat; a warp's NK partial dot
// products are summed over the lanes by a butterfly that halves the set of keys at each of the
// first log2 NK steps, so lane l ends with the score of key l >> (5 - log2 NK).  Each CTA leaves
// sum_j p_j v'_j and sum_j p_j in shared memory; CTA 0 of the cluster adds the chunks in order
// through distributed shared memory and writes out and lse.
template <int D>
struct DecCfg {
    static constexpr int DPL = D / 32;                  // features per lane
    static constexpr int KB = 4096 / D;                 // keys per tile: 32 (D = 128) or 64
    static constexpr int TILE_BYTES = KB * D * 2;       // 8 KB
    static constexpr int NS = 4;                        // ring stages (K and V' tile each)
    static constexpr int CONSUMERS = 4;
    static constexpr int THREADS = 32 * (CONSUMERS + 1);
    static constexpr int NK = KB / CONSUMERS;           // keys per consumer warp per tile: 8 or 16
    static constexpr int LOG_NK = NK == 8 ? 3 : 4;
    static constexpr int SMEM_RING = NS * 2 * TILE_BYTES;
    // ring | warp partials [CONSUMERS][D] | CTA partial [D + 1] | warp sums | barriers
    static constexpr int OFF_O = SMEM_RING;
    static constexpr int OFF_PART = OFF_O + CONSUMERS * D * 4;
    static constexpr int OFF_L = OFF_PART + (D + 4) * 4;
    static constexpr int OFF_BAR = OFF_L + 16;
    static constexpr int SMEM = OFF_BAR + 2 * NS * 8 + 1024;   // + alignment slack
};
constexpr int kDecodeMaxCluster = 8;

enum : unsigned int { kSiteDecFull = 70, kSiteDecEmpty = 71 };

// v[0..NK) per lane -> the lane's share of the sum over the warp of key (lane >> (5 - LOG_NK)).
template <int NK, int LOG_NK>
__device__ __forceinline__ float warp_sum_keys(float (&v)[NK], int lane) {
#pragma unroll
    for (int lvl = 0; lvl < LOG_NK; ++lvl) {
        const int n = NK >> (lvl + 1);
        const int m = 16 >> lvl;
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int j = 0; j < n; ++j) {
            const float mine = upper ? v[j + n] : v[j];
            const float other = upper ? v[j] : v[j + n];
            v[j] = mine + __shfl_xor_sync(0xffffffffu, other, m);
        }
    }
    float x = v[0];
#pragma unroll
    for (int m = 16 >> LOG_NK; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

struct DecParams {
    const __nv_bfloat16* q;      // (B*H, D) raw q of the new tokens (qhat is formed here)
    double rope_base, eps;
    int pos;                     // position of the new tokens
    __nv_bfloat16* out;          // (B*H, D)
    float* lse;                  // (B*H) or null
    const int* doc_start;        // (B) or null
    int H, Hkv, Tmax;
    int lo;                      // first window position
    int n_keys;                  // window keys: positions lo .. lo + n_keys - 1
    int tiles_per_chunk;         // KB-key tiles of each chunk (CTA); chunk c = tiles [c t, (c + 1) t)
    float c1, c2, m0;            // p = 2^(s c1 - c2); lse = m0 + ln sum p
    unsigned long long wait_limit_ns;
};

// tm_k, tm_v: the caches (B, Tmax, Hkv, D) as 3-D {D, Hkv, B * Tmax}, box {D, 1, KB}.
template <int D>
__global__ void __launch_bounds__(DecCfg<D>::THREADS) decode_attn_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                                         const __grid_constant__ CUtensorMap tm_v,
                                                                         const DecParams p) {
    using C = DecCfg<D>;
    constexpr int DPL = C::DPL, NK = C::NK, KB = C::KB;
    extern __shared__ __align__(1024) uint8_t dsmem[];
    uint8_t* smem = dsmem + ((1024u - (smem_u32(dsmem) & 1023u)) & 1023u);
    uint8_t* ring = smem;                                          // stage s: K at 2 s T, V' at (2 s + 1) T
    float* s_o = reinterpret_cast<float*>(smem + C::OFF_O);
    float* s_part = reinterpret_cast<float*>(smem + C::OFF_PART);
    float* s_l = reinterpret_cast<float*>(smem + C::OFF_L);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + C::NS;
    __shared__ float4 s_tab32[D / 2];
    __shared__ double2 s_tab64[D / 2];
    __shared__ __align__(16) __nv_bfloat16 s_qh[D];

    const int warp = (int)(threadIdx.x >> 5), lane = (int)(threadIdx.x & 31u);
    const uint32_t rank = cluster_ctarank(), n_ranks = cluster_nctarank();
    const int row = (int)(blockIdx.x / n_ranks);                   // b*H + h
    const int b = row / p.H, h = row - b * p.H;
    const int hk = h / (p.H / p.Hkv);
    // window-relative key range of this CTA, past the document start when there is one
    const int jmin = p.doc_start != nullptr ? max(0, min(__ldg(p.doc_start + b), p.lo + p.n_keys - 1) - p.lo) : 0;
    const int n_tiles = (p.n_keys + KB - 1) / KB;
    const int t_end = min((int)(rank + 1) * p.tiles_per_chunk, n_tiles);
    const int t_begin = max((int)rank * p.tiles_per_chunk, jmin / KB);
    const int key_begin = max((int)rank * p.tiles_per_chunk * KB, jmin);
    const int key_end = min((int)(rank + 1) * p.tiles_per_chunk * KB, p.n_keys);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), C::CONSUMERS);
        }
        fence_barrier_init();
    }
    __syncthreads();
    bool ok = true;
    if (warp == C::CONSUMERS) {
        // producer: one thread issues the tile loads
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const int y0 = b * p.Tmax + p.lo;
            for (int t = t_begin, i = 0; t < t_end; ++t, ++i) {
                const int s = i % C::NS;
                // the last tile holds the new token's key and value, written by the prologue kernel
                if (t == n_tiles - 1) grid_dependency_wait();
                if (i >= C::NS && !mbar_wait(smem_u32(empty + s), (uint32_t)((i / C::NS) - 1) & 1u, p.wait_limit_ns,
                                             kSiteDecEmpty)) {
                    ok = false;
                    break;
                }
                const uint32_t bar = smem_u32(full + s);
                mbar_arrive_expect_tx(bar, 2u * C::TILE_BYTES);
                tma_load_3d(smem_u32(ring + (2 * s) * C::TILE_BYTES), &tm_k, bar, 0, hk, y0 + t * KB);
                tma_load_3d(smem_u32(ring + (2 * s + 1) * C::TILE_BYTES), &tm_v, bar, 0, hk, y0 + t * KB);
            }
        }
    } else {
        // qhat of this row, formed here while the first tiles load: the RoPE row of `pos` (one
        // entry per thread of the first D/2), then the prologue's exact-rounding rotation and
        // RMS on warp 0 (D/8 lanes per row; the other lanes compute copies), as the prefill and
        // token prologues do, so qhat is bit-identical to theirs.
        if ((int)threadIdx.x < D / 2) {
            const int i = (int)threadIdx.x;
            const double theta = pow(p.rope_base, -2.0 * (double)i / (double)D);
            double sn, cs;
            sincos((double)p.pos * theta, &sn, &cs);
            float c_hi, c_lo, s_hi, s_lo;
            rope_split(cs, c_hi, c_lo);
            rope_split(sn, s_hi, s_lo);
            s_tab32[i] = make_float4(c_hi, c_lo, s_hi, s_lo);
            s_tab64[i] = make_double2(cs, sn);
        }
        asm volatile("bar.sync 1, %0;" ::"r"(32 * C::CONSUMERS) : "memory");
        if (warp == 0) {
            constexpr int TPR = D / 8;
            const int c = lane % TPR, i0 = 4 * c;
            const __nv_bfloat16* qr = p.q + (long long)row * D;
            const uint2 lo_raw = ldg_stream8(qr + i0), hi_raw = ldg_stream8(qr + D / 2 + i0);
            float4 cs4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) cs4[e] = s_tab32[i0 + e];
            uint2 o_lo, o_hi;
            rope_rms_exact4<D>(lo_raw, hi_raw, cs4, s_tab64 + i0, p.eps, o_lo, o_hi);
            if (lane < TPR) {
                *reinterpret_cast<uint2*>(s_qh + i0) = o_lo;
                *reinterpret_cast<uint2*>(s_qh + D / 2 + i0) = o_hi;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(32 * C::CONSUMERS) : "memory");
        float q[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) q[e] = __bfloat162float(s_qh[lane * DPL + e]);
        float o[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[e] = 0.f;
        float l = 0.f;
        for (int t = t_begin, i = 0; t < t_end; ++t, ++i) {
            const int s = i % C::NS;
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(full + s), (uint32_t)(i / C::NS) & 1u, p.wait_limit_ns,
                                                   kSiteDecFull))) {
                ok = false;
                break;
            }
            const int k0 = t * KB + warp * NK;                     // window-relative key of this warp's key 0
            const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(ring + (2 * s) * C::TILE_BYTES) +
                                      (warp * NK) * D + lane * DPL;
            const __nv_bfloat16* vt = reinterpret_cast<const __nv_bfloat16*>(ring + (2 * s + 1) * C::TILE_BYTES) +
                                      (warp * NK) * D + lane * DPL;
            float part[NK];
#pragma unroll
            for (int k = 0; k < NK; ++k) {
                Raw<DPL> rk;
                rk.load(kt + k * D);
                float kf[DPL];
                rk.unpack(kf);
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc = fmaf(q[e], kf[e], acc);
                part[k] = acc;
            }
            const float sc = warp_sum_keys<NK, C::LOG_NK>(part, lane);
            const int my_key = k0 + (lane >> (5 - C::LOG_NK));
            const bool visible = my_key >= key_begin && my_key < key_end;
            // masked keys: probability exactly 0 whatever the cache holds there
            const float pr = visible ? ex2_approx(fmaf(sc, p.c1, -p.c2)) : 0.f;
            if ((lane & ((1 << (5 - C::LOG_NK)) - 1)) == 0) l += pr;
#pragma unroll
            for (int k = 0; k < NK; ++k) {
                const float pk = __shfl_sync(0xffffffffu, pr, k << (5 - C::LOG_NK));
                const int key = k0 + k;
                if (key < key_begin || key >= key_end) continue;   // warp-uniform
                Raw<DPL> rv;
                rv.load(vt + k * D);
                float vf[DPL];
                rv.unpack(vf);
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[e] = fmaf(pk, vf[e], o[e]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(empty + s));
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) l += __shfl_xor_sync(0xffffffffu, l, m);
#pragma unroll
        for (int e = 0; e < DPL; ++e) s_o[warp * D + lane * DPL + e] = o[e];
        if (lane == 0) s_l[warp] = l;
    }
    __syncthreads();
    // this CTA's partial, warps added in a fixed order
    if (threadIdx.x < D) {
        const int d = (int)threadIdx.x;
        s_part[d] = (s_o[d] + s_o[D + d]) + (s_o[2 * D + d] + s_o[3 * D + d]);
    }
    if (threadIdx.x == D) s_part[D] = (s_l[0] + s_l[1]) + (s_l[2] + s_l[3]);
    cluster_sync_all();
    if (rank == 0 && threadIdx.x <= D) {
        const int d = (int)threadIdx.x;
        float acc = 0.f;
        for (uint32_t r = 0; r < n_ranks; ++r) acc += ld_shared_cluster_f32(s_part + d, r);
        float lsum = acc;
        if (d < D) {
            lsum = 0.f;
            for (uint32_t r = 0; r < n_ranks; ++r) lsum += ld_shared_cluster_f32(s_part + D, r);
            p.out[(long long)row * D + d] = __float2bfloat16_rn(acc / lsum);
        } else if (p.lse != nullptr) {
            p.lse[row] = p.m0 + logf(lsum);
        }
    }
    // peers keep their shared memory until CTA 0 has read it
    cluster_sync_all();
    (void)ok;
}

}  // namespace swa
