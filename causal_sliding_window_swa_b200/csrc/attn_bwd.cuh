// attn_bwd.cuh -- gradient of the causal sliding-window attention layer on the sm_100a tensor cores.
//
// The layer ("Let's reproduce GPT-2 (124M)" notes, section 3; intelliparadigm "GPT-2 for $73",
// sections 2.2 and 3.2; PaperWeekly repost, "Value Embeddings" paragraph) is
//   qhat, khat = rms(rope(q)), rms(rope(k));  v' = v + 2 sigmoid(x[:32] . Wg) ve;
//   out_i = sum_{j in J_i} P_ij v'_j,  P_ij = exp(s_ij - lse_i),  s_ij = qhat_i . khat_j / sqrt(D),
//   J_i = { j : 0 <= i - j < W }.
// For the loss sum(dout * out) + sum(dlse * lse) the chain rule gives, per visible pair,
//   dP_ij = dout_i . v'_j,  dS_ij = P_ij (dP_ij - (delta_i - dlse_i)),  delta_i = dout_i . out_i,
//   dqhat_i = sum_j dS_ij khat_j / sqrt(D),  dkhat_j = sum_i dS_ij qhat_i / sqrt(D),
//   dv'_j = sum_i P_ij dout_i,
// and then the prologue in reverse (RMS, RoPE, gate).  The softmax is rebuilt from the saved
// log-sum-exp, so no running maximum or sum is needed.
//
// Kernels, in launch order (after the forward prologue has recomputed qhat, khat, v'):
//   bwd_rowstat_kernel    per query row: (lse log2 e, delta - dlse), padded to whole tiles
//                         with (+inf, 0) so that rows past T get P = 0.
//   attn_bwd_dq_kernel    one 128-row query tile per item: S = Q K^T (two buffers in tensor
//                         memory) and dP = dO V'^T from shared-memory operands, dS by 16 warps,
//                         dQ += dS K with dS fed from tensor memory and K read MN-major; the next
//                         tile's S is computed while the warps work on this one.
//   attn_bwd_dkv_kernel   one 128-row key tile per item, over every query tile (and, under
//                         grouped-query attention, every query head of the group) that sees it:
//                         S^T = K Q^T and dP^T = V' dO^T from shared memory; the 16 warps write
//                         P^T first and dS^T second, so that dV += P^T dO and the next S^T run
//                         while dS^T is formed, and dK += dS^T Q and the next dP^T while the next
//                         P^T is.
//   Both tensor-core kernels end each item with the prologue in reverse for their rows: dq (dk)
//   = RoPE^T applied to the RMS backward of dqhat (dkhat), with the row sums exchanged between
//   the four threads of a row; dv = dv', dve = g dv', dz = (dv' . ve) g (1 - g / 2).
//   bwd_gate_x_kernel, bwd_wg_partial_kernel, bwd_wg_final_kernel
//                         dgate_x = dz Wg^T and dWg = gate_x^T dz (fixed summation order).
// The two tensor-core kernels use seven products per (query tile, key tile) pair instead of
// five so that neither needs fp32 atomics: dQ is owned by the query-tile kernel, dK and dV by the
// key-tile kernel.  The tensor-core operand forms here are A from tensor memory (bf16 pairs written
// by the warps, as the forward feeds P) or from shared memory (K-major, 128-byte swizzle), and B
// K-major or MN-major from shared memory.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace swa {

// 1-D bulk copy global -> shared memory, completing `bytes` on the mbarrier.  Both addresses
// 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

template <int D>
struct BwdCfg {
    static constexpr int NCHUNK = D / 64;              // 128-byte swizzle chunks per row
    static constexpr int CHUNK_BYTES = 128 * 128;      // 128 rows x 128 B
    static constexpr int TILE_BYTES = 128 * D * 2;     // one 128 x D bf16 tile
    static constexpr int SMEM_BAR = 512;
    static constexpr int THREADS = 576;
    static constexpr int SOFTMAX_THREADS = 512;
    static constexpr uint32_t TMEM_COLS = 512;
    // query-tile kernel: Q | dO | NS-stage ring of K and V' tiles | barriers
    static constexpr int DQ_NS = (D == 128) ? 4 : 10;
    static constexpr int DQ_RED = 2 * 4 * 128 * 8;      // row-sum exchange, two buffers of [4][128] float2
    static constexpr int THETA_BYTES = 512;            // theta_i, fp64, i < D / 2
    static constexpr int DQ_SMEM = 2 * TILE_BYTES + DQ_NS * TILE_BYTES + SMEM_BAR + DQ_RED + THETA_BYTES;
    static constexpr uint32_t DQ_COL_S = 0;            // S(0) | S(1), each then dS as bf16 pairs
    static constexpr uint32_t DQ_COL_DP = 256;
    static constexpr uint32_t DQ_COL_DQ = 384;         // D fp32 columns
    // key-tile kernel: K | V' | NS stages of (Q tile, dO tile, 128 row statistics) | barriers
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES + 1024;
    static constexpr int KV_NS = (D == 128) ? 2 : 5;
    static constexpr int KV_RED = 2 * 4 * 128 * 16;     // row-sum exchange, two buffers of [4][128] float4
    static constexpr int KV_SMEM = 2 * TILE_BYTES + KV_NS * STAGE_BYTES + SMEM_BAR + KV_RED + THETA_BYTES;
    static constexpr uint32_t KV_COL_ST = 0;           // S^T, then P^T as bf16 pairs
    static constexpr uint32_t KV_COL_DPT = 128;        // dP^T, then dS^T as bf16 pairs
    static constexpr uint32_t KV_COL_DV = 256;
    static constexpr uint32_t KV_COL_DK = 256 + D;
    static_assert(DQ_COL_DQ + D <= TMEM_COLS, "query-tile kernel exceeds tensor memory");
    static_assert(KV_COL_DK + D <= TMEM_COLS, "key-tile kernel exceeds tensor memory");
    static_assert(DQ_SMEM <= 227 * 1024 && KV_SMEM <= 227 * 1024, "shared memory per CTA");
};

struct BwdParams {
    int B, T, H, Hkv, G;   // G = H / Hkv query heads per key/value head
    int W;                 // effective window, 1..T
    int n_tiles;           // ceil(T / 128): query tiles = key tiles
    int Tp;                // n_tiles * 128, the row-statistics stride
    int n_items;
    int chunk_bh;          // (b, head) slices per scheduling chunk
    float c1;              // log2(e) / sqrt(D): raw score -> log2 units
    float inv_sqrt_d;
    const float2* rowstat; // (B, H, Tp): (lse log2 e, delta - dlse); padding rows (+inf, 0)
    // the prologue in reverse, applied in the epilogues
    const __nv_bfloat16* xq;   // (B, T, H, D) raw q
    const __nv_bfloat16* xk;   // (B, T, Hkv, D) raw k
    const __nv_bfloat16* ve;   // (B, T, Hkv, D) value embedding, or null
    const float2* gate;        // (B, T, Hkv) gate as (g_hi, g_lo), or null
    double rope_base;          // theta_i = rope_base^(-2 i / D)
    float eps;
    __nv_bfloat16* dq;         // (B, T, H, D)
    __nv_bfloat16* dk;         // (B, T, Hkv, D)
    __nv_bfloat16* dv;         // (B, T, Hkv, D)
    __nv_bfloat16* dve;        // (B, T, Hkv, D), value-embedding layers
    float* dz;                 // (B, T, Hkv): dL/dz of the gate's logit, value-embedding layers
    int* sched;            // [0] next item, [1] CTAs done; zero before the launch, reset after
    unsigned long long wait_limit_ns;
    const int* dstart;     // (B, T) first position of each position's document, or null (no mask)
    const int* dend;       // (B, T) last position of each position's document, or null
};

// Wait sites recorded in the status word on timeout (distinct from the forward's).
enum : unsigned int {
    kSiteBwdQFull = 40, kSiteBwdQEmpty = 41, kSiteBwdKvFull = 42, kSiteBwdKvEmpty = 43,
    kSiteBwdSFull = 44, kSiteBwdPFull = 45, kSiteBwdOFull = 46, kSiteBwdOEmpty = 47,
    kSiteBwdItem = 48, kSiteBwdDrain = 49, kSiteBwdStage = 50, kSiteBwdRed = 51
};

// Query-tile item: tile [q0, q0 + 127] of (b, h) and the key tiles lo..hi of its band; order as
// in the forward (chunks of (b, h) slices, heaviest tiles first inside a chunk).
struct BwdQItem {
    int b, h, q0, lo, hi;
};

__device__ __forceinline__ BwdQItem bwd_q_item(const BwdParams& p, int it) {
    BwdQItem m;
    const int per_chunk = p.chunk_bh * p.n_tiles;
    const int chunk = it / per_chunk;
    const int rem = it - chunk * per_chunk;
    const int first_bh = chunk * p.chunk_bh;
    const int n_bh = min(p.chunk_bh, p.B * p.H - first_bh);
    const int qt = p.n_tiles - 1 - rem / n_bh;
    const int bh = first_bh + rem % n_bh;
    m.b = bh / p.H;
    m.h = bh - m.b * p.H;
    m.q0 = qt * 128;
    m.lo = max(0, m.q0 - p.W + 1) / 128;
    m.hi = min(m.q0 + 127, p.T - 1) / 128;
    // Document mask: keys before the first row's document start are seen by no row of the tile.
    if (p.dstart != nullptr) m.lo = max(m.lo, p.dstart[(long long)m.b * p.T + m.q0] / 128);
    return m;
}

// Key-tile item: tile [k0, k0 + 127] of (b, hk); the queries that see it lie in
// [k0, k0 + 127 + W - 1], query tiles lo..hi, for each of the G query heads hk G .. hk G + G - 1.
// Under the causal mask the first key tiles are seen by the most queries, so they go first.
struct BwdKvItem {
    int b, hk, k0, lo, hi;
};

__device__ __forceinline__ BwdKvItem bwd_kv_item(const BwdParams& p, int it) {
    BwdKvItem m;
    const int per_chunk = p.chunk_bh * p.n_tiles;
    const int chunk = it / per_chunk;
    const int rem = it - chunk * per_chunk;
    const int first_bh = chunk * p.chunk_bh;
    const int n_bh = min(p.chunk_bh, p.B * p.Hkv - first_bh);
    const int kt = rem / n_bh;
    const int bh = first_bh + rem % n_bh;
    m.b = bh / p.Hkv;
    m.hk = bh - m.b * p.Hkv;
    m.k0 = kt * 128;
    m.lo = kt;
    m.hi = min(m.k0 + 127 + p.W - 1, p.T - 1) / 128;
    // Document mask: queries past the last key's document end see no key of the tile.
    if (p.dend != nullptr) m.hi = min(m.hi, p.dend[(long long)m.b * p.T + min(m.k0 + 127, p.T - 1)] / 128);
    return m;
}

// Byte offset (>> 4) of k-step kk (16 elements of the contraction) inside a K-major tile: 32 bytes
// inside a 128-byte swizzle chunk, chunks CHUNK_BYTES apart.
template <int D>
__device__ __forceinline__ uint64_t kmajor_step(int kk) {
    return (uint64_t)(((kk >> 2) * BwdCfg<D>::CHUNK_BYTES + (kk & 3) * 32) >> 4);
}

// ------------------------------------------------------------------- epilogue helpers
// An epilogue thread owns NP = D / 8 rotation pairs of one row, i in [i0, i0 + NP) with
// i0 = NP * (output quarter): elements i and i + D/2, so the rotation needs no other thread; the
// row sums are exchanged through shared memory between the four threads of the row.

template <int NP>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NP]) {
    if constexpr (NP == 16)
        tmem_ld16(taddr, r);
    else
        tmem_ld8(taddr, r);
}

// NP consecutive bf16 at p (16-byte aligned) -> fp32.
template <int NP>
__device__ __forceinline__ void load_bf16_row(const __nv_bfloat16* p, float (&x)[NP]) {
#pragma unroll
    for (int q = 0; q < NP / 8; ++q) {
        const uint4 u = *reinterpret_cast<const uint4*>(p + 8 * q);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[8 * q + 2 * e] = __uint_as_float(w[e] << 16);
            x[8 * q + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    }
}

// The same load kept packed (NP / 2 registers) until unpack_bf16_row.
template <int NP>
__device__ __forceinline__ void load_bf16_raw(const __nv_bfloat16* p, uint4 (&u)[NP / 8]) {
#pragma unroll
    for (int q = 0; q < NP / 8; ++q) u[q] = *reinterpret_cast<const uint4*>(p + 8 * q);
}

template <int NP>
__device__ __forceinline__ void unpack_bf16_row(const uint4 (&u)[NP / 8], float (&x)[NP]) {
#pragma unroll
    for (int q = 0; q < NP / 8; ++q) {
        const uint32_t w[4] = {u[q].x, u[q].y, u[q].z, u[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[8 * q + 2 * e] = __uint_as_float(w[e] << 16);
            x[8 * q + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    }
}

template <int NP>
__device__ __forceinline__ void store_bf16_row(__nv_bfloat16* p, const float (&y)[NP]) {
#pragma unroll
    for (int q = 0; q < NP / 8; ++q)
        *reinterpret_cast<uint4*>(p + 8 * q) =
            make_uint4(pack_bf16x2(y[8 * q], y[8 * q + 1]), pack_bf16x2(y[8 * q + 2], y[8 * q + 3]),
                       pack_bf16x2(y[8 * q + 4], y[8 * q + 5]), pack_bf16x2(y[8 * q + 6], y[8 * q + 7]));
}

// RMS backward then RoPE transposed, for this thread's pairs: g = dL/dxhat (ga at i, gb at
// i + D/2), x the raw input row, tab its RoPE (cos, sin).  With u = R^T g (ua = ga c + gb s,
// ub = gb c - ga s), the row sums ss = sum x^2 and xu = sum x . u give
// dx = r u - r^3 (xu / D) x, r = 1 / sqrt(ss / D + eps).  Phase 1 returns this thread's partial
// sums and fills ua, ub; phase 2 takes the row's sums.
// cos and sin of t theta_i for this thread's NP frequencies (theta from shared memory, fp64): the
// angle is formed and reduced to [-pi, pi] in fp64 (error below 1e-11), then evaluated on the
// special-function unit in fp32 (absolute error about 1e-6, well inside the gradient's tolerance).
template <int NP>
__device__ __forceinline__ void rope_cs_fast(int t, const double* __restrict__ theta, float (&c)[NP], float (&sn)[NP]) {
    constexpr double kTwoPi = 6.283185307179586;
    constexpr double kInvTwoPi = 0.15915494309189535;
#pragma unroll
    for (int e = 0; e < NP; ++e) {
        const double a = (double)t * theta[e];
        const double red = fma(-rint(a * kInvTwoPi), kTwoPi, a);
        __sincosf((float)red, &sn[e], &c[e]);
    }
}

template <int NP>
__device__ __forceinline__ void rms_rope_bwd_partial(const float (&ga)[NP], const float (&gb)[NP],
                                                     const float (&xa)[NP], const float (&xb)[NP],
                                                     const float (&cc)[NP], const float (&ssn)[NP], float (&ua)[NP],
                                                     float (&ub)[NP], float& ss, float& xu) {
    ss = 0.f;
    xu = 0.f;
#pragma unroll
    for (int e = 0; e < NP; ++e) {
        const float c = cc[e], sn = ssn[e];
        ua[e] = ga[e] * c + gb[e] * sn;
        ub[e] = gb[e] * c - ga[e] * sn;
        ss += xa[e] * xa[e] + xb[e] * xb[e];
        xu += xa[e] * ua[e] + xb[e] * ub[e];
    }
}

template <int NP>
__device__ __forceinline__ void rms_rope_bwd_finish(float ss, float xu, int D, float eps, const float (&ua)[NP],
                                                    const float (&ub)[NP], float (&xa)[NP], float (&xb)[NP]) {
    const float rr = rsqrtf(ss / (float)D + eps);
    const float coef = rr * rr * rr * xu / (float)D;
#pragma unroll
    for (int e = 0; e < NP; ++e) {
        xa[e] = rr * ua[e] - coef * xa[e];
        xb[e] = rr * ub[e] - coef * xb[e];
    }
}

// ------------------------------------------------------------------- row statistics

// delta = dout . out over D (fp32) for every (b, h, t), t < Tp, stored with the log-sum-exp in
// log2 units.  L = D / 8 consecutive lanes share a row, one 16-byte load of each tensor per lane.
// Block 0 also zeroes the scheduler counters of the two tensor-core kernels.
template <int D>
__global__ void bwd_rowstat_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                                   const float* __restrict__ lse, const float* __restrict__ dlse,
                                   float2* __restrict__ rowstat, int B, int T, int H, int Tp,
                                   int* __restrict__ sched4) {
    if (blockIdx.x == 0 && threadIdx.x < 4) sched4[threadIdx.x] = 0;
    constexpr int L = D / 8;   // lanes per row: 16 or 8
    const int sub = threadIdx.x & (L - 1);
    const int n = B * H * Tp;
    const int f = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) / L);
    // every lane of a row group takes the same branch; groups are aligned inside the warp
    const bool live = f < n;
    const int t = live ? f % Tp : 0;
    const int bh = live ? f / Tp : 0;
    float acc = 0.f;
    if (live && t < T) {
        const int h = bh % H;
        const int b = bh / H;
        const long long e0 = (((long long)b * T + t) * H + h) * D + sub * 8;
        const uint4 a = *reinterpret_cast<const uint4*>(out + e0);
        const uint4 g = *reinterpret_cast<const uint4*>(dout + e0);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int w = 0; w < 4; ++w)
            acc += __uint_as_float(aw[w] << 16) * __uint_as_float(gw[w] << 16) +
                   __uint_as_float(aw[w] & 0xffff0000u) * __uint_as_float(gw[w] & 0xffff0000u);
    }
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (live && sub == 0) {
        if (t >= T) {
            rowstat[f] = make_float2(__int_as_float(0x7f800000), 0.f);
        } else {
            const long long li = (long long)bh * T + t;
            const float gl = dlse ? dlse[li] : 0.f;
            rowstat[f] = make_float2(lse[li] * 1.4426950408889634f, acc - gl);
        }
    }
}

// ------------------------------------------------------------------ query-tile kernel (dQ)

// Per item (query tile of (b, h), key tiles lo..hi; g counts tiles over the CTA's items):
//   S(g) = Q K_j^T into S buffer g % 2 and dP(g) = dO V_j^T, both with Q / dO and K / V' read
//   from shared memory; the 16 warps turn S(g), dP(g) into dS(g) (bf16, over S(g)'s columns);
//   dQ += dS(g) K_j with K read MN-major.  Issue order of the MMA thread:
//     S(0) dP(0) | S(1) [wait dS(0)] dP(1) dQ(0) | S(2) [wait dS(1)] dP(2) dQ(1) | ...
//   so while the warps work on tile g the tensor pipe runs dQ(g - 1) and S(g + 1), and only dP(g + 1)
//   waits for them.  S(g + 2) overwrites the buffer whose dS(g) the dQ(g) product issued just
//   before it reads (products execute in issue order).
template <int D, bool DOC = false>
__global__ void __launch_bounds__(576, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr int NS = C::DQ_NS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0u) {   // uniform: every thread leaves before any barrier
        if (threadIdx.x == 0) record_error(kErrLayout, 0);
        return;
    }
    uint8_t* sQ = smem_raw;
    uint8_t* sdO = sQ + C::TILE_BYTES;
    uint8_t* sKV = sdO + C::TILE_BYTES;          // NS tiles: K_j, V'_j alternately
    uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NS * C::TILE_BYTES);
    uint64_t* b_qfull = bars + 0;                // Q and dO tiles landed
    uint64_t* b_qempty = bars + 1;               // the item's products are done reading them
    uint64_t* b_ofull = bars + 2;                // dQ of the item complete
    uint64_t* b_oempty = bars + 3;               // dQ read by the epilogue
    uint64_t* b_mdrain = bars + 4;
    uint64_t* b_itfull = bars + 5;               // [2]
    uint64_t* b_itempty = bars + 7;              // [2]
    uint64_t* b_sfull = bars + 9;                // S(g) and dP(g) complete
    uint64_t* b_pfull = bars + 10;               // dS(g) written to tensor memory
    uint64_t* b_kvfull = bars + 11;              // [NS]
    uint64_t* b_kvempty = bars + 11 + NS;        // [NS]
    uint64_t* b_red = bars + 11 + 2 * NS;        // [2] row sums of an epilogue written
    int* s_item = reinterpret_cast<int*>(bars + 13 + 2 * NS);   // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_item + 2);
    float2* s_red = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(bars) + C::SMEM_BAR);   // [2][4][128]
    double* s_theta = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(s_red) + C::DQ_RED);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr int kMmaWarp = 0;
    constexpr int kProducerWarp = 1;
    constexpr int kSoftmaxWarp0 = 2;
    constexpr uint32_t kItemConsumers = 1 + 16;

    if (threadIdx.x == 32) {
        mbar_init(smem_u32(b_qfull), 1);
        mbar_init(smem_u32(b_qempty), 1);
        mbar_init(smem_u32(b_ofull), 1);
        mbar_init(smem_u32(b_oempty), C::SOFTMAX_THREADS);
        mbar_init(smem_u32(b_mdrain), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(b_itfull + i), 1);
            mbar_init(smem_u32(b_itempty + i), kItemConsumers);
        }
        mbar_init(smem_u32(b_sfull), 1);
        mbar_init(smem_u32(b_pfull), C::SOFTMAX_THREADS);
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(b_kvfull + s), 1);
            mbar_init(smem_u32(b_kvempty + s), 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(smem_u32(b_red + i), C::SOFTMAX_THREADS);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + D / 2)
        s_theta[threadIdx.x - 64] = pow(p.rope_base, -2.0 * (double)(threadIdx.x - 64) / (double)D);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = p.wait_limit_ns;

    if (warp == kProducerWarp) {
        // ========================= scheduler + TMA producer =========================
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t filled_phase[NS];
            bool filled[NS];
            for (int s = 0; s < NS; ++s) filled[s] = false, filled_phase[s] = 0;
            uint32_t q_uses = 0;
            bool ok = true;
            auto load_kv = [&](const CUtensorMap* tm, const BwdQItem& m, int j) -> bool {
                if (!mbar_wait(smem_u32(b_kvempty + stage), phase ^ 1u, lim, kSiteBwdKvEmpty)) return false;
                const uint32_t fb = smem_u32(b_kvfull + stage);
                mbar_arrive_expect_tx(fb, (uint32_t)C::TILE_BYTES);
                for (int ch = 0; ch < C::NCHUNK; ++ch)
                    tma_load_4d(smem_u32(sKV + stage * C::TILE_BYTES + ch * C::CHUNK_BYTES), tm, fb, ch * 64,
                                m.h / p.G, j * 128, m.b);
                filled[stage] = true;
                filled_phase[stage] = phase;
                if (++stage == (uint32_t)NS) {
                    stage = 0;
                    phase ^= 1u;
                }
                return true;
            };
            for (uint32_t k = 0; ok; ++k) {
                int it = atomicAdd(p.sched, 1);
                if (it >= p.n_items) it = -1;
                const uint32_t slot = k & 1u;
                if (!(ok = mbar_wait(smem_u32(b_itempty + slot), ((k >> 1) & 1u) ^ 1u, lim, kSiteBwdItem))) break;
                s_item[slot] = it;
                mbar_arrive(smem_u32(b_itfull + slot));
                if (it < 0) break;
                const BwdQItem m = bwd_q_item(p, it);
                // Warm L2 with this item's Q and dO while the previous item finishes with its own.
                for (int ch = 0; ch < C::NCHUNK; ++ch) {
                    tma_prefetch_4d(&tm_q, ch * 64, m.h, m.q0, m.b);
                    tma_prefetch_4d(&tm_do, ch * 64, m.h, m.q0, m.b);
                }
                if (q_uses > 0 && !(ok = mbar_wait(smem_u32(b_qempty), (q_uses - 1) & 1u, lim, kSiteBwdQEmpty)))
                    break;
                {
                    const uint32_t qb = smem_u32(b_qfull);
                    mbar_arrive_expect_tx(qb, 2u * (uint32_t)C::TILE_BYTES);
                    for (int ch = 0; ch < C::NCHUNK; ++ch) {
                        tma_load_4d(smem_u32(sQ + ch * C::CHUNK_BYTES), &tm_q, qb, ch * 64, m.h, m.q0, m.b);
                        tma_load_4d(smem_u32(sdO + ch * C::CHUNK_BYTES), &tm_do, qb, ch * 64, m.h, m.q0, m.b);
                    }
                    ++q_uses;
                }
                // The MMA thread's order: K_j, then V'_j, for each key tile j.
                for (int j = m.lo; ok && j <= m.hi; ++j) ok = load_kv(&tm_k, m, j) && load_kv(&tm_v, m, j);
            }
            if (ok && atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
                p.sched[0] = 0;
                p.sched[1] = 0;
            }
            if (q_uses > 0) mbar_wait(smem_u32(b_qfull), (q_uses - 1) & 1u, lim, kSiteBwdDrain);
            for (int s = 0; s < NS; ++s)
                if (filled[s]) mbar_wait(smem_u32(b_kvfull + s), filled_phase[s], lim, kSiteBwdDrain);
        }
    } else if (warp == kMmaWarp) {
        // ============================== MMA issuer ==============================
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);   // S, dP: N = 128 keys
            constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, true);     // dQ: B = K MN-major
            const uint64_t a_q = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t a_do = smem_desc_sw128(smem_u32(sdO), 16, 1024);
            const uint64_t dkv_k = smem_desc_sw128(smem_u32(sKV), 16, 1024);
            const uint64_t dkv_mn = smem_desc_sw128(smem_u32(sKV), C::CHUNK_BYTES, 1024);
            uint32_t stage = 0, phase = 0;
            uint32_t g = 0;       // tiles over this CTA's items: S buffer g & 1, barrier parities
            uint32_t uses = 0;    // items done
            auto acquire = [&](uint32_t& s) -> bool {
                s = stage;
                const bool r = mbar_wait(smem_u32(b_kvfull + stage), phase, lim, kSiteBwdKvFull);
                if (++stage == (uint32_t)NS) {
                    stage = 0;
                    phase ^= 1u;
                }
                return r;
            };
            auto s_mma = [&](uint32_t buf, uint32_t sk) {
                const uint64_t bk = dkv_k + (uint64_t)((sk * C::TILE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::DQ_COL_S + 128u * buf, a_q + kmajor_step<D>(kk), bk + kmajor_step<D>(kk), idesc_s,
                           kk > 0 ? 1u : 0u);
            };
            auto dp_mma = [&](uint32_t sv) {
                const uint64_t bv = dkv_k + (uint64_t)((sv * C::TILE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::DQ_COL_DP, a_do + kmajor_step<D>(kk), bv + kmajor_step<D>(kk), idesc_s,
                           kk > 0 ? 1u : 0u);
                mma_commit(smem_u32(b_sfull));
                mma_commit(smem_u32(b_kvempty + sv));
            };
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                const uint32_t slot = k & 1u;
                if (!(ok = mbar_wait(smem_u32(b_itfull + slot), (k >> 1) & 1u, lim, kSiteBwdItem))) break;
                const int it = s_item[slot];
                mbar_arrive(smem_u32(b_itempty + slot));
                if (it < 0) break;
                const BwdQItem m = bwd_q_item(p, it);
                if (!(ok = mbar_wait(smem_u32(b_qfull), uses & 1u, lim, kSiteBwdQFull))) break;
                const int n = m.hi - m.lo + 1;
                uint32_t sk_cur = 0, sk_next = 0, sv = 0;
                if (!(ok = acquire(sk_cur))) break;
                s_mma(g & 1u, sk_cur);
                if (!(ok = acquire(sv))) break;
                dp_mma(sv);
                for (int t = 0; ok && t < n; ++t) {
                    const bool more = t + 1 < n;
                    if (more) {
                        if (!(ok = acquire(sk_next))) break;
                        s_mma((g + 1u) & 1u, sk_next);
                    }
                    if (!(ok = mbar_wait(smem_u32(b_pfull), g & 1u, lim, kSiteBwdPFull))) break;
                    if (t == 0 && uses > 0 &&
                        !(ok = mbar_wait(smem_u32(b_oempty), (uses - 1) & 1u, lim, kSiteBwdOEmpty)))
                        break;
                    tc_fence_after();
                    if (more) {
                        if (!(ok = acquire(sv))) break;
                        dp_mma(sv);
                    }
                    // dQ += dS K_j: K = 128 keys in steps of 16; dS of keys 32 c + i at column
                    // 32 c + i / 2 of the tile's S buffer.
                    const uint64_t bkm = dkv_mn + (uint64_t)((sk_cur * C::TILE_BYTES) >> 4);
                    const uint32_t a_ds = tmem + C::DQ_COL_S + 128u * (g & 1u);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + C::DQ_COL_DQ, a_ds + (kk >> 1) * 32 + (kk & 1) * 8,
                               bkm + (uint64_t)((kk * 16 * 128) >> 4), idesc_dq, (t > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(smem_u32(b_kvempty + sk_cur));
                    sk_cur = sk_next;
                    ++g;
                }
                if (!ok) break;
                mma_commit(smem_u32(b_qempty));
                mma_commit(smem_u32(b_ofull));
                ++uses;
            }
            mma_commit(smem_u32(b_mdrain));
            mbar_wait(smem_u32(b_mdrain), 0, lim, kSiteBwdDrain);
        }
        __syncwarp();
    } else {
        // ============================ dS + epilogue ============================
        const int cq = (warp - kSoftmaxWarp0) >> 2;   // key / output column quarter
        const int r = ((warp & 3) << 5) + lane;       // tile row = tensor-memory lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t g = 0, o_uses = 0;
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            const uint32_t slot = k & 1u;
            int it = 0;
            if (lane == 0) {
                ok = mbar_wait(smem_u32(b_itfull + slot), (k >> 1) & 1u, lim, kSiteBwdItem);
                it = s_item[slot];
                mbar_arrive(smem_u32(b_itempty + slot));
            }
            ok = __all_sync(0xffffffffu, ok);
            it = __shfl_sync(0xffffffffu, it, 0);
            if (!ok || it < 0) break;
            const BwdQItem m = bwd_q_item(p, it);
            const int qi = m.q0 + r;
            // the epilogue's raw q row, into L2 while the item's tiles are worked on
            if (cq < D / 64 && qi < p.T)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.xq + (((long long)m.b * p.T + qi) * p.H + m.h) * D + 64 * cq));
            // document mask: this row sees no key before its document's start
            const int ds = DOC ? __ldg(p.dstart + (long long)m.b * p.T + min(qi, p.T - 1)) : 0;
            const float2 rs = p.rowstat[((long long)m.b * p.H + m.h) * p.Tp + qi];
            const float nl = -rs.x, dl = rs.y;
            for (int j = m.lo; j <= m.hi; ++j, ++g) {
                const bool w = mbar_wait(smem_u32(b_sfull), g & 1u, lim, kSiteBwdSFull);
                ok = __all_sync(0xffffffffu, w);
                if (!ok) break;
                tc_fence_after();
                const int k0 = j * 128 + 32 * cq;
                uint32_t sv[2][16], dv[2][16], pk[16];
                const uint32_t colS = C::DQ_COL_S + 128u * (g & 1u) + 32u * (uint32_t)cq;
                const uint32_t colP = C::DQ_COL_DP + 32u * (uint32_t)cq;
                tmem_ld16(tmem + lane_base + colS, sv[0]);
                tmem_ld16(tmem + lane_base + colS + 16u, sv[1]);
                tmem_ld16(tmem + lane_base + colP, dv[0]);
                tmem_ld16(tmem + lane_base + colP + 16u, dv[1]);
                tmem_ld_wait();
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
#pragma unroll
                    for (int e = 0; e < 16; e += 2) {
                        const int kv = k0 + 16 * hb + e;
                        float p0 = ex2_approx(fmaf(__uint_as_float(sv[hb][e]), p.c1, nl));
                        float p1 = ex2_approx(fmaf(__uint_as_float(sv[hb][e + 1]), p.c1, nl));
                        if ((unsigned)(qi - kv) >= (unsigned)p.W || (DOC && kv < ds)) p0 = 0.f;
                        if ((unsigned)(qi - kv - 1) >= (unsigned)p.W || (DOC && kv + 1 < ds)) p1 = 0.f;
                        const float d0 = p0 * (__uint_as_float(dv[hb][e]) - dl);
                        const float d1 = p1 * (__uint_as_float(dv[hb][e + 1]) - dl);
                        pk[8 * hb + (e >> 1)] = pack_bf16x2(d0, d1);
                    }
                }
                tmem_st16(tmem + lane_base + colS, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(smem_u32(b_pfull));
            }
            if (!ok) break;
            // The raw q row (the epilogue's input that does not depend on dQ) is fetched while the
            // item's last dQ product runs.
            constexpr int NP = D / 8;
            const int i0 = NP * cq;
            const bool live = qi < p.T;
            const int qc = min(qi, p.T - 1);
            const long long roff = (((long long)m.b * p.T + qc) * p.H + m.h) * D;
            uint4 xra[NP / 8], xrb[NP / 8];
            load_bf16_raw<NP>(p.xq + roff + i0, xra);
            load_bf16_raw<NP>(p.xq + roff + D / 2 + i0, xrb);
            {
                const bool w = mbar_wait(smem_u32(b_ofull), o_uses & 1u, lim, kSiteBwdOFull);
                ok = __all_sync(0xffffffffu, w);
            }
            if (!ok) break;
            tc_fence_after();
            // dqhat of this thread's pairs (columns i0 .. and D/2 + i0 ..), then dq = RoPE^T of the
            // RMS backward (the prologue in reverse)
            uint32_t gau[NP], gbu[NP];
            tmem_ld_cols<NP>(tmem + lane_base + C::DQ_COL_DQ + (uint32_t)i0, gau);
            tmem_ld_cols<NP>(tmem + lane_base + C::DQ_COL_DQ + (uint32_t)(D / 2 + i0), gbu);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(smem_u32(b_oempty));
            const uint32_t e_idx = o_uses++;
            float xa[NP], xb[NP], cc[NP], sn[NP], ga[NP], gb[NP], ua[NP], ub[NP];
            unpack_bf16_row<NP>(xra, xa);
            unpack_bf16_row<NP>(xrb, xb);
            rope_cs_fast<NP>(qc, s_theta + i0, cc, sn);
#pragma unroll
            for (int e = 0; e < NP; ++e) {
                ga[e] = __uint_as_float(gau[e]) * p.inv_sqrt_d;
                gb[e] = __uint_as_float(gbu[e]) * p.inv_sqrt_d;
            }
            float ss, xu;
            rms_rope_bwd_partial<NP>(ga, gb, xa, xb, cc, sn, ua, ub, ss, xu);
            float2* red = s_red + (e_idx & 1u) * 512u;
            red[cq * 128 + r] = make_float2(ss, xu);
            mbar_arrive(smem_u32(b_red + (e_idx & 1u)));
            {
                const bool w = mbar_wait(smem_u32(b_red + (e_idx & 1u)), (e_idx >> 1) & 1u, lim, kSiteBwdRed);
                ok = __all_sync(0xffffffffu, w);
            }
            if (!ok) break;
            const float2 t0 = red[r], t1 = red[128 + r], t2 = red[256 + r], t3 = red[384 + r];
            rms_rope_bwd_finish<NP>((t0.x + t1.x) + (t2.x + t3.x), (t0.y + t1.y) + (t2.y + t3.y), D, p.eps, ua, ub,
                                    xa, xb);
            if (live) {
                store_bf16_row<NP>(p.dq + roff + i0, xa);
                store_bf16_row<NP>(p.dq + roff + D / 2 + i0, xb);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- key-tile kernel (dK, dV)

// Per item (key tile of (b, hk); steps s over the G query heads x query tiles that see it):
//   S^T(s) = K Q_s^T and dP^T(s) = V' dO_s^T (shared-memory operands), then the 16 warps in two
//   phases: A turns S^T into P^T (bf16, over S^T's columns; P stays in registers), B turns dP^T
//   into dS^T = P^T (dP^T - (delta - dlse)) (bf16, over dP^T's columns).  Issue order:
//     S^T(0) dP^T(0) | [P^T(0)] dV(0) S^T(1) [dS^T(0)] dK(0) dP^T(1) | [P^T(1)] dV(1) S^T(2) ...
//   so phase A of step s + 1 waits only for dV(s) and S^T(s + 1), and phase B for dK(s) and
//   dP^T(s + 1); each overwrite of a buffer follows, in issue order, the product that reads it.
template <int D, bool DOC = false>
__global__ void __launch_bounds__(576, 1)
    attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr int NS = C::KV_NS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0u) {
        if (threadIdx.x == 0) record_error(kErrLayout, 0);
        return;
    }
    uint8_t* sK = smem_raw;
    uint8_t* sV = sK + C::TILE_BYTES;
    uint8_t* sSt = sV + C::TILE_BYTES;           // NS stages: Q tile | dO tile | 128 x float2
    uint64_t* bars = reinterpret_cast<uint64_t*>(sSt + NS * C::STAGE_BYTES);
    uint64_t* b_kfull = bars + 0;                // K and V' tiles of the item landed
    uint64_t* b_kempty = bars + 1;               // the item's products are done with them
    uint64_t* b_ofull = bars + 2;
    uint64_t* b_oempty = bars + 3;
    uint64_t* b_mdrain = bars + 4;
    uint64_t* b_itfull = bars + 5;               // [2]
    uint64_t* b_itempty = bars + 7;              // [2]
    uint64_t* b_stready = bars + 9;              // S^T(s) complete
    uint64_t* b_dpready = bars + 10;             // dP^T(s) complete
    uint64_t* b_pready = bars + 11;              // P^T(s) written
    uint64_t* b_dsready = bars + 12;             // dS^T(s) written
    uint64_t* b_stfull = bars + 13;              // [NS]
    uint64_t* b_stempty = bars + 13 + NS;        // [NS]
    uint64_t* b_red = bars + 13 + 2 * NS;        // [2] row sums of an epilogue written
    int* s_item = reinterpret_cast<int*>(bars + 15 + 2 * NS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_item + 2);
    float4* s_red = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(bars) + C::SMEM_BAR);   // [2][4][128]
    double* s_theta = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(s_red) + C::KV_RED);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr int kMmaWarp = 0;
    constexpr int kProducerWarp = 1;
    constexpr int kSoftmaxWarp0 = 2;
    constexpr uint32_t kItemConsumers = 1 + 16;

    if (threadIdx.x == 32) {
        mbar_init(smem_u32(b_kfull), 1);
        mbar_init(smem_u32(b_kempty), 1);
        mbar_init(smem_u32(b_ofull), 1);
        mbar_init(smem_u32(b_oempty), C::SOFTMAX_THREADS);
        mbar_init(smem_u32(b_mdrain), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(b_itfull + i), 1);
            mbar_init(smem_u32(b_itempty + i), kItemConsumers);
        }
        mbar_init(smem_u32(b_stready), 1);
        mbar_init(smem_u32(b_dpready), 1);
        mbar_init(smem_u32(b_pready), C::SOFTMAX_THREADS);
        mbar_init(smem_u32(b_dsready), C::SOFTMAX_THREADS);
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(b_stfull + s), 1);
            mbar_init(smem_u32(b_stempty + s), 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(smem_u32(b_red + i), C::SOFTMAX_THREADS);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + D / 2)
        s_theta[threadIdx.x - 64] = pow(p.rope_base, -2.0 * (double)(threadIdx.x - 64) / (double)D);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = p.wait_limit_ns;

    if (warp == kProducerWarp) {
        // ========================= scheduler + TMA producer =========================
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t filled_phase[NS];
            bool filled[NS];
            for (int s = 0; s < NS; ++s) filled[s] = false, filled_phase[s] = 0;
            uint32_t kv_uses = 0;
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                int it = atomicAdd(p.sched, 1);
                if (it >= p.n_items) it = -1;
                const uint32_t slot = k & 1u;
                if (!(ok = mbar_wait(smem_u32(b_itempty + slot), ((k >> 1) & 1u) ^ 1u, lim, kSiteBwdItem))) break;
                s_item[slot] = it;
                mbar_arrive(smem_u32(b_itfull + slot));
                if (it < 0) break;
                const BwdKvItem m = bwd_kv_item(p, it);
                // Warm L2 with this item's K and V' while the previous item still uses its own.
                for (int ch = 0; ch < C::NCHUNK; ++ch) {
                    tma_prefetch_4d(&tm_k, ch * 64, m.hk, m.k0, m.b);
                    tma_prefetch_4d(&tm_v, ch * 64, m.hk, m.k0, m.b);
                }
                if (kv_uses > 0 && !(ok = mbar_wait(smem_u32(b_kempty), (kv_uses - 1) & 1u, lim, kSiteBwdKvEmpty)))
                    break;
                {
                    const uint32_t kb = smem_u32(b_kfull);
                    mbar_arrive_expect_tx(kb, 2u * (uint32_t)C::TILE_BYTES);
                    for (int ch = 0; ch < C::NCHUNK; ++ch) {
                        tma_load_4d(smem_u32(sK + ch * C::CHUNK_BYTES), &tm_k, kb, ch * 64, m.hk, m.k0, m.b);
                        tma_load_4d(smem_u32(sV + ch * C::CHUNK_BYTES), &tm_v, kb, ch * 64, m.hk, m.k0, m.b);
                    }
                    ++kv_uses;
                }
                for (int g = 0; ok && g < p.G; ++g) {
                    const int h = m.hk * p.G + g;
                    for (int i = m.lo; ok && i <= m.hi; ++i) {
                        if (!(ok = mbar_wait(smem_u32(b_stempty + stage), phase ^ 1u, lim, kSiteBwdStage))) break;
                        const uint32_t fb = smem_u32(b_stfull + stage);
                        uint8_t* base = sSt + stage * C::STAGE_BYTES;
                        mbar_arrive_expect_tx(fb, 2u * (uint32_t)C::TILE_BYTES + 1024u);
                        for (int ch = 0; ch < C::NCHUNK; ++ch) {
                            tma_load_4d(smem_u32(base + ch * C::CHUNK_BYTES), &tm_q, fb, ch * 64, h, i * 128, m.b);
                            tma_load_4d(smem_u32(base + C::TILE_BYTES + ch * C::CHUNK_BYTES), &tm_do, fb, ch * 64, h,
                                        i * 128, m.b);
                        }
                        bulk_load_1d(smem_u32(base + 2 * C::TILE_BYTES),
                                     p.rowstat + ((long long)m.b * p.H + h) * p.Tp + (long long)i * 128, 1024u, fb);
                        filled[stage] = true;
                        filled_phase[stage] = phase;
                        if (++stage == (uint32_t)NS) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            if (ok && atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
                p.sched[0] = 0;
                p.sched[1] = 0;
            }
            if (kv_uses > 0) mbar_wait(smem_u32(b_kfull), (kv_uses - 1) & 1u, lim, kSiteBwdDrain);
            for (int s = 0; s < NS; ++s)
                if (filled[s]) mbar_wait(smem_u32(b_stfull + s), filled_phase[s], lim, kSiteBwdDrain);
        }
    } else if (warp == kMmaWarp) {
        // ============================== MMA issuer ==============================
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);   // S^T, dP^T: N = 128 queries
            constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, true);      // dV, dK: B MN-major
            const uint64_t a_k = smem_desc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t a_v = smem_desc_sw128(smem_u32(sV), 16, 1024);
            const uint64_t b_kmaj = smem_desc_sw128(smem_u32(sSt), 16, 1024);
            const uint64_t b_mn = smem_desc_sw128(smem_u32(sSt), C::CHUNK_BYTES, 1024);
            uint32_t stage = 0, phase = 0;
            uint32_t g = 0, uses = 0;   // steps over this CTA's items (barrier parities); items done
            auto acquire = [&](uint32_t& sg) -> bool {
                sg = stage;
                const bool r = mbar_wait(smem_u32(b_stfull + stage), phase, lim, kSiteBwdStage);
                if (++stage == (uint32_t)NS) {
                    stage = 0;
                    phase ^= 1u;
                }
                return r;
            };
            auto st_mma = [&](uint32_t sg) {
                const uint64_t qoff = (uint64_t)((sg * C::STAGE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::KV_COL_ST, a_k + kmajor_step<D>(kk), b_kmaj + qoff + kmajor_step<D>(kk),
                           idesc_s, kk > 0 ? 1u : 0u);
                mma_commit(smem_u32(b_stready));
            };
            auto dpt_mma = [&](uint32_t sg) {
                const uint64_t dooff = (uint64_t)((sg * C::STAGE_BYTES + C::TILE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::KV_COL_DPT, a_v + kmajor_step<D>(kk), b_kmaj + dooff + kmajor_step<D>(kk),
                           idesc_s, kk > 0 ? 1u : 0u);
                mma_commit(smem_u32(b_dpready));
            };
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                const uint32_t slot = k & 1u;
                if (!(ok = mbar_wait(smem_u32(b_itfull + slot), (k >> 1) & 1u, lim, kSiteBwdItem))) break;
                const int it = s_item[slot];
                mbar_arrive(smem_u32(b_itempty + slot));
                if (it < 0) break;
                const BwdKvItem m = bwd_kv_item(p, it);
                if (!(ok = mbar_wait(smem_u32(b_kfull), uses & 1u, lim, kSiteBwdKvFull))) break;
                const int n_steps = p.G * (m.hi - m.lo + 1);
                uint32_t sg = 0, sg_next = 0;
                if (!(ok = acquire(sg))) break;
                st_mma(sg);
                dpt_mma(sg);
                for (int s = 0; ok && s < n_steps; ++s) {
                    const bool more = s + 1 < n_steps;
                    const uint64_t qoff = (uint64_t)((sg * C::STAGE_BYTES) >> 4);
                    const uint64_t dooff = (uint64_t)((sg * C::STAGE_BYTES + C::TILE_BYTES) >> 4);
                    if (!(ok = mbar_wait(smem_u32(b_pready), g & 1u, lim, kSiteBwdPFull))) break;
                    if (s == 0 && uses > 0 &&
                        !(ok = mbar_wait(smem_u32(b_oempty), (uses - 1) & 1u, lim, kSiteBwdOEmpty)))
                        break;
                    tc_fence_after();
                    // dV += P^T dO: K = 128 queries in steps of 16; P^T of queries 32 c + i at
                    // column 32 c + i / 2 of the S^T buffer.
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + C::KV_COL_DV, tmem + C::KV_COL_ST + (kk >> 1) * 32 + (kk & 1) * 8,
                               b_mn + dooff + (uint64_t)((kk * 16 * 128) >> 4), idesc_g, (s > 0 || kk > 0) ? 1u : 0u);
                    if (more) {
                        if (!(ok = acquire(sg_next))) break;
                        st_mma(sg_next);
                    }
                    if (!(ok = mbar_wait(smem_u32(b_dsready), g & 1u, lim, kSiteBwdSFull))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + C::KV_COL_DK, tmem + C::KV_COL_DPT + (kk >> 1) * 32 + (kk & 1) * 8,
                               b_mn + qoff + (uint64_t)((kk * 16 * 128) >> 4), idesc_g, (s > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(smem_u32(b_stempty + sg));
                    if (more) dpt_mma(sg_next);
                    sg = sg_next;
                    ++g;
                }
                if (!ok) break;
                mma_commit(smem_u32(b_ofull));
                mma_commit(smem_u32(b_kempty));
                ++uses;
            }
            mma_commit(smem_u32(b_mdrain));
            mbar_wait(smem_u32(b_mdrain), 0, lim, kSiteBwdDrain);
        }
        __syncwarp();
    } else {
        // ========================= P^T, dS^T + epilogue =========================
        const int cq = (warp - kSoftmaxWarp0) >> 2;   // query / output column quarter
        const int r = ((warp & 3) << 5) + lane;       // key row = tensor-memory lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t colS = C::KV_COL_ST + 32u * (uint32_t)cq;
        const uint32_t colP = C::KV_COL_DPT + 32u * (uint32_t)cq;
        uint32_t stage = 0, phase = 0;
        uint32_t g = 0, o_uses = 0;
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            const uint32_t slot = k & 1u;
            int it = 0;
            if (lane == 0) {
                ok = mbar_wait(smem_u32(b_itfull + slot), (k >> 1) & 1u, lim, kSiteBwdItem);
                it = s_item[slot];
                mbar_arrive(smem_u32(b_itempty + slot));
            }
            ok = __all_sync(0xffffffffu, ok);
            it = __shfl_sync(0xffffffffu, it, 0);
            if (!ok || it < 0) break;
            const BwdKvItem m = bwd_kv_item(p, it);
            const int key = m.k0 + r;
            // the epilogue's raw k and value-embedding rows, into L2 while the item is worked on
            if (cq < D / 64 && key < p.T) {
                const long long o = (((long long)m.b * p.T + key) * p.Hkv + m.hk) * D + 64 * cq;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.xk + o));
                if (p.ve != nullptr) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.ve + o));
            }
            // document mask: no query past this key's document end sees it
            const int de = DOC ? __ldg(p.dend + (long long)m.b * p.T + min(key, p.T - 1)) : 0;
            const int nq = m.hi - m.lo + 1;
            const int n_steps = p.G * nq;
            for (int s = 0; s < n_steps; ++s, ++g) {
                const int i = m.lo + s % nq;
                const uint32_t sg = stage;
                // Phase A: S^T(s) is complete, and (through the stage's own barrier, still in this
                // phase) so is the copy of its row statistics.
                bool w = mbar_wait(smem_u32(b_stready), g & 1u, lim, kSiteBwdSFull);
                w = w && mbar_wait(smem_u32(b_stfull + sg), phase, lim, kSiteBwdStage);
                ok = __all_sync(0xffffffffu, w);
                if (!ok) break;
                if (++stage == (uint32_t)NS) {
                    stage = 0;
                    phase ^= 1u;
                }
                tc_fence_after();
                const float2* rs = reinterpret_cast<const float2*>(sSt + sg * C::STAGE_BYTES + 2 * C::TILE_BYTES) + 32 * cq;
                const int qc0 = i * 128 + 32 * cq;      // first query column of this thread
                float pv[32];
                {
                    uint32_t sv[2][16], pp[16];
                    tmem_ld16(tmem + lane_base + colS, sv[0]);
                    tmem_ld16(tmem + lane_base + colS + 16u, sv[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float2 r0 = rs[c], r1 = rs[c + 1];
                        float p0 = ex2_approx(fmaf(__uint_as_float(sv[c >> 4][c & 15]), p.c1, -r0.x));
                        float p1 = ex2_approx(fmaf(__uint_as_float(sv[c >> 4][(c & 15) + 1]), p.c1, -r1.x));
                        if ((unsigned)(qc0 + c - key) >= (unsigned)p.W || (DOC && qc0 + c > de)) p0 = 0.f;
                        if ((unsigned)(qc0 + c + 1 - key) >= (unsigned)p.W || (DOC && qc0 + c + 1 > de)) p1 = 0.f;
                        pv[c] = p0;
                        pv[c + 1] = p1;
                        pp[c >> 1] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(tmem + lane_base + colS, pp);
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(smem_u32(b_pready));
                // Phase B: dP^T(s) is complete.
                w = mbar_wait(smem_u32(b_dpready), g & 1u, lim, kSiteBwdSFull);
                ok = __all_sync(0xffffffffu, w);
                if (!ok) break;
                tc_fence_after();
                {
                    uint32_t dv[2][16], pd[16];
                    tmem_ld16(tmem + lane_base + colP, dv[0]);
                    tmem_ld16(tmem + lane_base + colP + 16u, dv[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float d0 = pv[c] * (__uint_as_float(dv[c >> 4][c & 15]) - rs[c].y);
                        const float d1 = pv[c + 1] * (__uint_as_float(dv[c >> 4][(c & 15) + 1]) - rs[c + 1].y);
                        pd[c >> 1] = pack_bf16x2(d0, d1);
                    }
                    tmem_st16(tmem + lane_base + colP, pd);
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(smem_u32(b_dsready));
            }
            if (!ok) break;
            // dK and dV' of this thread's pairs (columns i0 .. and D/2 + i0 ..); then the prologue in
            // reverse: dk = RoPE^T of the RMS backward (raw k row), dv = dv', and on value-embedding
            // layers dve = g dv' and dz = (dv' . ve) g (1 - g / 2), the derivative of g = 2 sigmoid(z)
            // being 2 sigmoid (1 - sigmoid).  The raw k row (an input that does not depend on the
            // products) is fetched while the item's last products run.
            constexpr int NP = D / 8;
            const int i0 = NP * cq;
            const bool live = key < p.T;
            const int kc = min(key, p.T - 1);
            const long long rrow = ((long long)m.b * p.T + kc) * p.Hkv + m.hk;
            const long long roff = rrow * D;
            uint4 xra[NP / 8], xrb[NP / 8], era[NP / 8], erb[NP / 8];
            load_bf16_raw<NP>(p.xk + roff + i0, xra);
            load_bf16_raw<NP>(p.xk + roff + D / 2 + i0, xrb);
            float g = 0.f;
            {
                const bool w = mbar_wait(smem_u32(b_ofull), o_uses & 1u, lim, kSiteBwdOFull);
                ok = __all_sync(0xffffffffu, w);
            }
            if (!ok) break;
            tc_fence_after();
            // dV' first: dv = dv', dve = g dv' and this thread's part of dv' . ve
            float dvve = 0.f;
            {
                uint32_t vau[NP], vbu[NP];
                tmem_ld_cols<NP>(tmem + lane_base + C::KV_COL_DV + (uint32_t)i0, vau);
                tmem_ld_cols<NP>(tmem + lane_base + C::KV_COL_DV + (uint32_t)(D / 2 + i0), vbu);
                tmem_ld_wait();
                float va[NP], vb[NP];
#pragma unroll
                for (int e = 0; e < NP; ++e) {
                    va[e] = __uint_as_float(vau[e]);
                    vb[e] = __uint_as_float(vbu[e]);
                }
                if (live) {
                    store_bf16_row<NP>(p.dv + roff + i0, va);
                    store_bf16_row<NP>(p.dv + roff + D / 2 + i0, vb);
                }
                if (p.ve != nullptr) {
                    load_bf16_raw<NP>(p.ve + roff + i0, era);
                    load_bf16_raw<NP>(p.ve + roff + D / 2 + i0, erb);
                    const float2 gg = p.gate[rrow];
                    g = gg.x + gg.y;
                    float ea[NP], eb[NP];
                    unpack_bf16_row<NP>(era, ea);
                    unpack_bf16_row<NP>(erb, eb);
#pragma unroll
                    for (int e = 0; e < NP; ++e) {
                        dvve += va[e] * ea[e] + vb[e] * eb[e];
                        va[e] *= g;
                        vb[e] *= g;
                    }
                    if (live) {
                        store_bf16_row<NP>(p.dve + roff + i0, va);
                        store_bf16_row<NP>(p.dve + roff + D / 2 + i0, vb);
                    }
                }
            }
            // then dK: dk = RoPE^T of the RMS backward, with the raw k row
            float xa[NP], xb[NP], ua[NP], ub[NP];
            float ss, xu;
            {
                uint32_t kau[NP], kbu[NP];
                tmem_ld_cols<NP>(tmem + lane_base + C::KV_COL_DK + (uint32_t)i0, kau);
                tmem_ld_cols<NP>(tmem + lane_base + C::KV_COL_DK + (uint32_t)(D / 2 + i0), kbu);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(smem_u32(b_oempty));
                unpack_bf16_row<NP>(xra, xa);
                unpack_bf16_row<NP>(xrb, xb);
                float ga[NP], gb[NP];
#pragma unroll
                for (int e = 0; e < NP; ++e) {
                    ga[e] = __uint_as_float(kau[e]) * p.inv_sqrt_d;
                    gb[e] = __uint_as_float(kbu[e]) * p.inv_sqrt_d;
                }
                float cc[NP], sn[NP];
                rope_cs_fast<NP>(kc, s_theta + i0, cc, sn);
                rms_rope_bwd_partial<NP>(ga, gb, xa, xb, cc, sn, ua, ub, ss, xu);
            }
            const uint32_t e_idx = o_uses++;
            float4* red = s_red + (e_idx & 1u) * 512u;
            red[cq * 128 + r] = make_float4(ss, xu, dvve, 0.f);
            mbar_arrive(smem_u32(b_red + (e_idx & 1u)));
            {
                const bool w = mbar_wait(smem_u32(b_red + (e_idx & 1u)), (e_idx >> 1) & 1u, lim, kSiteBwdRed);
                ok = __all_sync(0xffffffffu, w);
            }
            if (!ok) break;
            const float4 t0 = red[r], t1 = red[128 + r], t2 = red[256 + r], t3 = red[384 + r];
            rms_rope_bwd_finish<NP>((t0.x + t1.x) + (t2.x + t3.x), (t0.y + t1.y) + (t2.y + t3.y), D, p.eps, ua, ub,
                                    xa, xb);
            if (live) {
                store_bf16_row<NP>(p.dk + roff + i0, xa);
                store_bf16_row<NP>(p.dk + roff + D / 2 + i0, xb);
                if (p.ve != nullptr && cq == 0) p.dz[rrow] = ((t0.z + t1.z) + (t2.z + t3.z)) * g * (1.f - 0.5f * g);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------- the gate in reverse

// dgate_x[bt, c] = sum_hk dz[bt, hk] Wg[c, hk]: one thread per (bt, c).
__global__ void bwd_gate_x_kernel(const float* __restrict__ dz, const __nv_bfloat16* __restrict__ Wg,
                                  float* __restrict__ dgx, long long n_bt, int Hkv) {
    const long long n = n_bt * 32;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long bt = idx >> 5;
        const int c = (int)(idx & 31);
        float acc = 0.f;
        for (int hk = 0; hk < Hkv; ++hk) acc += dz[bt * Hkv + hk] * __bfloat162float(Wg[c * Hkv + hk]);
        dgx[idx] = acc;
    }
}

// dWg in two passes with a fixed order: block blk sums rows [blk R, blk R + R) into
// part[blk][c Hkv + hk]; the final pass gives each output one block, whose threads add strided
// partials and then combine them by a tree in shared memory.
__global__ void bwd_wg_partial_kernel(const float* __restrict__ dz, const __nv_bfloat16* __restrict__ gate_x,
                                      float* __restrict__ part, long long n_bt, int Hkv, int rows_per_block) {
    const int n = 32 * Hkv;
    const long long r0 = (long long)blockIdx.x * rows_per_block;
    const long long r1 = min(r0 + rows_per_block, n_bt);
    for (int idx = threadIdx.x; idx < n; idx += blockDim.x) {
        const int c = idx / Hkv;
        const int hk = idx - c * Hkv;
        float acc = 0.f;
#pragma unroll 8
        for (long long bt = r0; bt < r1; ++bt) acc += dz[bt * Hkv + hk] * __bfloat162float(gate_x[bt * 32 + c]);
        part[(long long)blockIdx.x * n + idx] = acc;
    }
}

// One block of 256 threads per output index.
__global__ void bwd_wg_final_kernel(const float* __restrict__ part, float* __restrict__ dWg, int n_blocks, int n) {
    __shared__ float red[256];
    const int idx = blockIdx.x;
    float acc = 0.f;
    for (int b = threadIdx.x; b < n_blocks; b += 256) acc += part[(long long)b * n + idx];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) dWg[idx] = red[0];
}

}  // namespace swa
