// attn_fwd.cuh -- causal sliding-window attention forward on the sm_100a tensor cores.
//
// What it computes ("Let's reproduce GPT-2 (124M)" notes, section 3 and section 19;
// intelliparadigm "GPT-2 for $73", section 3.2):
//   out[b,i,h,:] = sum_{j in J_i} softmax_j(qhat_i . khat_j / sqrt(D)) v'_j,
//   J_i = { j : 0 <= i - j < W },  lse[b,h,i] = ln sum_{j in J_i} exp(qhat_i . khat_j / sqrt(D)),
// on the RMS-normalised, rotated qhat/khat and the gated v' that the prologue wrote.
//
// Work item: two adjacent 128-row query tiles of one (b, h).  The item walks the 128-row
// key/value tiles that intersect its window band [q0 - W + 1, q0 + 255]; tiles outside the band
// are never loaded.  The kernel is persistent: one CTA per SM takes items from a global counter
// (ordered in L2-sized chunks of (b, h) slices, heaviest first inside a chunk) until none is left.
// Warp roles (320 threads):
//   warp  0    TMEM allocator and the single thread that issues tcgen05.mma
//   warp  1    scheduler + TMA producer: Q tiles, then K_j, V_j through an NS-stage mbarrier ring
//   warps 2-5  softmax + epilogue for query tile 0 (warp w owns rows 32 (w % 4) .. +31: TMEM lanes)
//   warps 6-9  softmax + epilogue for query tile 1
// Tensor memory (512 columns): S0 | S1 (128 fp32 columns each) | O0 | O1 (D columns each).
// P (bf16) is written over the first 64 columns of its S buffer and fed to the PV product
// straight from tensor memory.
//
// Softmax offset.  After the RMS QK-norm every |qhat . khat| / sqrt(D) is at most
// sqrt(D) (1 + 2^-8)^2 (bf16 rounding of the unit-RMS vectors), so exp(s - M0) with the fixed
// offset M0 = sqrt(D) (1 + 2^-6) lies in (e^(-2 M0), 1].  The online-softmax recurrence of the
// pages (running max m, l' = e^(m - m') l + sum e^(s - m'), accumulator rescaled by e^(m - m'))
// is run with m pinned at that upper bound: every rescale factor is exactly 1, so the
// accumulator never needs correcting and each row's sum stays in its own thread.  The result is
// the same softmax (it is shift invariant) and lse = M0 + ln l exactly.  The output is divided
// by the sum of the bf16-rounded P that the PV product actually multiplied, so the weights it
// applies sum to one (a row with one visible key returns that key's v' unchanged); the LSE uses
// the unrounded sum.  P is rounded to bf16 toward zero (one byte-permute per pair); because the
// normaliser is the sum of the same rounded values, the rounding bias cancels in the weights.
// One exponential in four is evaluated by a polynomial on the FMA pipe to offload the MUFU unit.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace swa {

template <int D>
struct FwdCfg {
    static constexpr int BM = 128;                     // query rows per tile (MMA M)
    static constexpr int BN = 128;                     // key rows per tile
    static constexpr int NCHUNK = D / 64;              // 128-byte swizzle chunks per row
    static constexpr int CHUNK_BYTES = 128 * 128;      // 128 rows x 128 B
    static constexpr int TILE_BYTES = 128 * D * 2;     // one 128 x D bf16 tile
    static constexpr int NS = (D == 128) ? 5 : 10;     // K/V ring depth
    static constexpr int SMEM_Q = 2 * TILE_BYTES;
    static constexpr int SMEM_KV = NS * TILE_BYTES;
    static constexpr int SMEM_BAR = 512;
    static constexpr int SMEM_TOTAL = 1024 /*alignment slack*/ + SMEM_Q + SMEM_KV + SMEM_BAR;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
    static constexpr int THREADS = 320;
};

struct FwdParams {
    int B, T, H;
    int W;                 // effective window, 1..T
    int n_pairs;           // ceil(ceil(T/128)/2)
    int n_items;           // n_pairs * H * B
    int chunk_bh;          // (b, h) slices per scheduling chunk
    float c1;              // log2(e) / sqrt(D): raw score -> log2 units
    float c2;              // M0 * log2(e)
    float m0;              // M0 (natural-log units), added back into the LSE
    __nv_bfloat16* out;    // (B,T,H,D)
    float* lse;            // (B,H,T) or null
    int* sched;            // [0] next item, [1] CTAs done; zero before the launch, reset after
    unsigned long long wait_limit_ns;
};

// Wait sites recorded in the status word on timeout.
enum : unsigned int {
    kSiteQFull = 1, kSiteKvEmpty = 2, kSiteKvFull = 3, kSiteSFull = 4, kSitePFull = 5,
    kSiteOFull = 6, kSiteDrain = 7, kSiteQEmpty = 8, kSiteOEmpty = 9, kSiteItem = 10
};

// Decoded work item.
template <int D>
struct Item {
    int b, h;
    int q0[2], lo_t[2], hi_t[2];
    bool valid[2];
    int lo, hi;
    __device__ __forceinline__ bool active(int g, int j) const {
        return valid[g] && j >= lo_t[g] && j <= hi_t[g];
    }
};

// Item order: chunks of `chunk_bh` (b, h) slices (their K/V fit in L2 together); inside a chunk,
// query-tile pairs from the last (heaviest under the causal mask) to the first.
template <int D>
__device__ __forceinline__ Item<D> decode_item(const FwdParams& p, int it) {
    using C = FwdCfg<D>;
    Item<D> m;
    const int per_chunk = p.chunk_bh * p.n_pairs;
    const int chunk = it / per_chunk;
    const int rem = it - chunk * per_chunk;
    const int first_bh = chunk * p.chunk_bh;
    const int n_bh = min(p.chunk_bh, p.B * p.H - first_bh);
    const int pair = p.n_pairs - 1 - rem / n_bh;
    const int bh = first_bh + rem % n_bh;
    m.b = bh / p.H;
    m.h = bh - m.b * p.H;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        m.q0[g] = (2 * pair + g) * C::BM;
        m.valid[g] = m.q0[g] < p.T;
        const int first_key = max(0, m.q0[g] - p.W + 1);
        const int last_key = min(m.q0[g] + C::BM - 1, p.T - 1);
        m.lo_t[g] = first_key / C::BN;
        m.hi_t[g] = last_key / C::BN;
    }
    m.lo = m.lo_t[0];
    m.hi = m.valid[1] ? m.hi_t[1] : m.hi_t[0];
    return m;
}

// One pair of raw scores -> P = 2^(s c1 - c2) on MUFU; accumulates the exact and the rounded
// sums (paired fp32) and returns the two P values as bf16 (toward zero) in one word.
__device__ __forceinline__ uint32_t softmax_pair_mufu(uint32_t s0, uint32_t s1, uint64_t c1x2,
                                                      uint64_t nc2x2, uint64_t& l2, uint64_t& lr2) {
    uint32_t w;
    asm("{\n\t"
        ".reg .b64 x, pp, tt;\n\t"
        ".reg .f32 x0, x1, p0, p1;\n\t"
        "mov.b64 x, {%3, %4};\n\t"
        "fma.rn.f32x2 x, x, %5, %6;\n\t"
        "mov.b64 {x0, x1}, x;\n\t"
        "ex2.approx.ftz.f32 p0, x0;\n\t"
        "ex2.approx.ftz.f32 p1, x1;\n\t"
        "mov.b64 pp, {p0, p1};\n\t"
        "add.rn.f32x2 %1, %1, pp;\n\t"
        "and.b64 tt, pp, 0xffff0000ffff0000;\n\t"
        "add.rn.f32x2 %2, %2, tt;\n\t"
        "prmt.b32 %0, p0, p1, 0x7632;\n\t"
        "}"
        : "=r"(w), "+l"(l2), "+l"(lr2)
        : "r"(s0), "r"(s1), "l"(c1x2), "l"(nc2x2));
    return w;
}

// Same, with 2^x evaluated on the FMA pipe: x = n + f, n = round(x) by the 1.5 * 2^23 shifter,
// f in [-1/2, 1/2]; 2^f by a degree-3 polynomial whose coefficients minimise the maximum
// relative error on that interval (Remez exchange fitted for this library, 7.5e-5 in fp32);
// 2^n applied by adding n to the exponent field.  Valid for x in [-126, 0].
struct PolyConsts {
    uint64_t shift, nshift, neg1, c3, c2, c1, c0;
};

__device__ __forceinline__ uint32_t softmax_pair_poly(uint32_t s0, uint32_t s1, uint64_t c1x2,
                                                      uint64_t nc2x2, const PolyConsts& k,
                                                      uint64_t& l2, uint64_t& lr2) {
    uint32_t w;
    asm("{\n\t"
        ".reg .b64 x, t, n, f, q, tt;\n\t"
        ".reg .b32 q0, q1, t0, t1;\n\t"
        "mov.b64 x, {%3, %4};\n\t"
        "fma.rn.f32x2 x, x, %5, %6;\n\t"
        "add.rn.f32x2 t, x, %7;\n\t"
        "add.rn.f32x2 n, t, %8;\n\t"
        "fma.rn.f32x2 f, n, %9, x;\n\t"
        "fma.rn.f32x2 q, %10, f, %11;\n\t"
        "fma.rn.f32x2 q, q, f, %12;\n\t"
        "fma.rn.f32x2 q, q, f, %13;\n\t"
        "mov.b64 {q0, q1}, q;\n\t"
        "mov.b64 {t0, t1}, t;\n\t"
        "shl.b32 t0, t0, 23;\n\t"
        "shl.b32 t1, t1, 23;\n\t"
        "add.s32 q0, q0, t0;\n\t"
        "add.s32 q1, q1, t1;\n\t"
        "mov.b64 q, {q0, q1};\n\t"
        "add.rn.f32x2 %1, %1, q;\n\t"
        "and.b64 tt, q, 0xffff0000ffff0000;\n\t"
        "add.rn.f32x2 %2, %2, tt;\n\t"
        "prmt.b32 %0, q0, q1, 0x7632;\n\t"
        "}"
        : "=r"(w), "+l"(l2), "+l"(lr2)
        : "r"(s0), "r"(s1), "l"(c1x2), "l"(nc2x2), "l"(k.shift), "l"(k.nshift), "l"(k.neg1),
          "l"(k.c3), "l"(k.c2), "l"(k.c1), "l"(k.c0));
    return w;
}

template <int D>
__global__ void __maxnreg__(168)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;                          // 2 tiles
    uint8_t* sKV = smem + C::SMEM_Q;             // NS tiles
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_Q + C::SMEM_KV);
    uint64_t* b_qfull = bars + 0;                // [2]
    uint64_t* b_qempty = bars + 2;               // [2]
    uint64_t* b_sfull = bars + 4;                // [2]
    uint64_t* b_pfull = bars + 6;                // [2]
    uint64_t* b_ofull = bars + 8;                // [2]
    uint64_t* b_oempty = bars + 10;              // [2]
    uint64_t* b_itfull = bars + 12;              // [2] scheduler slots
    uint64_t* b_itempty = bars + 14;             // [2]
    uint64_t* b_mdrain = bars + 16;              // MMA thread's final drain
    uint64_t* b_kvfull = bars + 17;              // [NS]
    uint64_t* b_kvempty = bars + 17 + C::NS;     // [NS]
    int* s_item = reinterpret_cast<int*>(bars + 17 + 2 * C::NS);   // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_item + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // The MMA thread gets the lowest warp id: among ready warps the issue logic tends to favour
    // lower ids, and the tensor core idles whenever this thread waits for an issue slot.
    constexpr int kMmaWarp = 0;
    constexpr int kProducerWarp = 1;
    constexpr int kSoftmaxWarp0 = 2;             // warps 2-5: tile 0, warps 6-9: tile 1
    constexpr uint32_t kItemConsumers = 1 + 8;   // the MMA thread and lane 0 of each softmax warp

    if (threadIdx.x == 32) {
        for (int g = 0; g < 2; ++g) {
            mbar_init(smem_u32(b_qfull + g), 1);
            mbar_init(smem_u32(b_qempty + g), 1);
            mbar_init(smem_u32(b_sfull + g), 1);
            mbar_init(smem_u32(b_pfull + g), 128);
            mbar_init(smem_u32(b_ofull + g), 1);
            mbar_init(smem_u32(b_oempty + g), 128);
            mbar_init(smem_u32(b_itfull + g), 1);
            mbar_init(smem_u32(b_itempty + g), kItemConsumers);
        }
        mbar_init(smem_u32(b_mdrain), 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(smem_u32(b_kvfull + s), 1);
            mbar_init(smem_u32(b_kvempty + s), 1);
        }
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = p.wait_limit_ns;

    if (warp == kProducerWarp) {
        // ========================= scheduler + TMA producer =========================
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t filled_phase[C::NS];
            bool filled[C::NS];
            for (int s = 0; s < C::NS; ++s) filled[s] = false, filled_phase[s] = 0;
            uint32_t q_uses[2] = {0u, 0u};
            bool ok = true;
            auto load_kv = [&](const CUtensorMap* tm, const Item<D>& m, int j) -> bool {
                if (!mbar_wait(smem_u32(b_kvempty + stage), phase ^ 1u, lim, kSiteKvEmpty)) return false;
                const uint32_t fb = smem_u32(b_kvfull + stage);
                mbar_arrive_expect_tx(fb, (uint32_t)C::TILE_BYTES);
                for (int ch = 0; ch < C::NCHUNK; ++ch)
                    tma_load_4d(smem_u32(sKV + stage * C::TILE_BYTES + ch * C::CHUNK_BYTES), tm, fb, ch * 64,
                                m.h, j * C::BN, m.b);
                filled[stage] = true;
                filled_phase[stage] = phase;
                if (++stage == (uint32_t)C::NS) {
                    stage = 0;
                    phase ^= 1u;
                }
                return true;
            };
            auto load_q = [&](const Item<D>& m, int g) -> bool {
                if (q_uses[g] > 0 &&
                    !mbar_wait(smem_u32(b_qempty + g), (q_uses[g] - 1) & 1u, lim, kSiteQEmpty))
                    return false;
                const uint32_t qb = smem_u32(b_qfull + g);
                mbar_arrive_expect_tx(qb, (uint32_t)C::TILE_BYTES);
                for (int ch = 0; ch < C::NCHUNK; ++ch)
                    tma_load_4d(smem_u32(sQ + g * C::TILE_BYTES + ch * C::CHUNK_BYTES), &tm_q, qb, ch * 64,
                                m.h, m.q0[g], m.b);
                ++q_uses[g];
                return true;
            };
            for (uint32_t k = 0; ok; ++k) {
                int it = atomicAdd(p.sched, 1);
                if (it >= p.n_items) it = -1;
                const uint32_t slot = k & 1u;
                if (!(ok = mbar_wait(smem_u32(b_itempty + slot), ((k >> 1) & 1u) ^ 1u, lim, kSiteItem))) break;
                s_item[slot] = it;
                mbar_arrive(smem_u32(b_itfull + slot));
                if (it < 0) break;
                const Item<D> m = decode_item<D>(p, it);
                // Warm L2 with this item's query tiles while the previous item finishes.
                for (int g = 0; g < 2; ++g)
                    if (m.valid[g])
                        for (int ch = 0; ch < C::NCHUNK; ++ch) tma_prefetch_4d(&tm_q, ch * 64, m.h, m.q0[g], m.b);
                // Order: Q0, K_lo, Q1, V_lo, then K/V of the rest, so tile 0 can start before tile 1.
                ok = load_q(m, 0) && load_kv(&tm_k, m, m.lo) && (!m.valid[1] || load_q(m, 1)) &&
                     load_kv(&tm_v, m, m.lo);
                for (int j = m.lo + 1; ok && j <= m.hi; ++j) ok = load_kv(&tm_k, m, j) && load_kv(&tm_v, m, j);
            }
            // The last CTA to run out of items resets the counters for the next launch.
            if (ok && atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
                p.sched[0] = 0;
                p.sched[1] = 0;
            }
            // Drain: every copy this thread started has landed before the CTA may exit.
            for (int g = 0; g < 2; ++g)
                if (q_uses[g] > 0) mbar_wait(smem_u32(b_qfull + g), (q_uses[g] - 1) & 1u, lim, kSiteDrain);
            for (int s = 0; s < C::NS; ++s)
                if (filled[s]) mbar_wait(smem_u32(b_kvfull + s), filled_phase[s], lim, kSiteDrain);
        }
    } else if (warp == kMmaWarp) {
        // ============================== MMA issuer ==============================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, C::BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dkv = smem_desc_sw128(smem_u32(sKV), 16, 1024);
            const uint64_t dv = smem_desc_sw128(smem_u32(sKV), C::CHUNK_BYTES, 1024);
            uint32_t stage = 0, phase = 0;
            uint32_t p_phase[2] = {0u, 0u};
            uint32_t uses[2] = {0u, 0u};     // items in which each query tile was valid
            // K/V ring slot; the data arrived by TMA, so the barrier wait alone orders the reads.
            auto acquire = [&](uint32_t& s) -> bool {
                s = stage;
                const bool r = mbar_wait(smem_u32(b_kvfull + stage), phase, lim, kSiteKvFull);
                if (++stage == (uint32_t)C::NS) {
                    stage = 0;
                    phase ^= 1u;
                }
                return r;
            };
            // S_g = Q_g K^T : M=128, N=BN, K=D in steps of 16 (32 bytes inside a 128-byte swizzle
            // chunk; the descriptor start address advances in 16-byte units).
            auto issue_s = [&](int g, uint32_t sk) {
                const uint64_t da = dq + (uint64_t)((g * C::TILE_BYTES) >> 4);
                const uint64_t db = dkv + (uint64_t)((sk * C::TILE_BYTES) >> 4);
                const uint32_t d = tmem + (g == 0 ? C::COL_S0 : C::COL_S1);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4;
                    mma_ss(d, da + off, db + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O_g += P_g V : M=128, N=D, K=BN in steps of 16 key rows.  P from tensor memory
            // (8 columns of packed bf16 pairs per step), V MN-major from shared memory.
            auto issue_pv = [&](int g, uint32_t sv, bool acc) {
                const uint32_t pa = tmem + (g == 0 ? C::COL_S0 : C::COL_S1);
                const uint32_t d = tmem + (g == 0 ? C::COL_O0 : C::COL_O1);
                const uint64_t db = dv + (uint64_t)((sv * C::TILE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ts(d, pa + kk * 8, db + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                           (acc || kk > 0) ? 1u : 0u);
            };
            // S_g(j), then release Q_g once its last S product of the item is issued.
            auto s_step = [&](const Item<D>& m, int g, uint32_t sk, int j) {
                issue_s(g, sk);
                mma_commit(smem_u32(b_sfull + g));
                if (j == m.hi_t[g]) mma_commit(smem_u32(b_qempty + g));
            };
            // PV_g(j); the item's first PV of a tile waits until the previous epilogue of that tile
            // has read its O.
            auto pv_step = [&](const Item<D>& m, int g, uint32_t sv, int j) -> bool {
                if (!mbar_wait(smem_u32(b_pfull + g), p_phase[g], lim, kSitePFull)) return false;
                p_phase[g] ^= 1u;
                if (j == m.lo_t[g] && uses[g] > 0 &&
                    !mbar_wait(smem_u32(b_oempty + g), (uses[g] - 1) & 1u, lim, kSiteOEmpty))
                    return false;
                tc_fence_after();
                issue_pv(g, sv, j > m.lo_t[g]);
                if (j == m.hi_t[g]) mma_commit(smem_u32(b_ofull + g));
                return true;
            };

            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                const uint32_t slot = k & 1u;
                if (!(ok = mbar_wait(smem_u32(b_itfull + slot), (k >> 1) & 1u, lim, kSiteItem))) break;
                const int it = s_item[slot];
                mbar_arrive(smem_u32(b_itempty + slot));
                if (it < 0) break;
                const Item<D> m = decode_item<D>(p, it);
                // Tile 0 starts as soon as its Q and the first K are in; tile 1 waits for its Q
                // only when its first product is due.
                uint32_t sk = 0;
                if (!(ok = mbar_wait(smem_u32(b_qfull + 0), uses[0] & 1u, lim, kSiteQFull))) break;
                if (!(ok = acquire(sk))) break;
                if (m.active(0, m.lo)) s_step(m, 0, sk, m.lo);
                if (m.valid[1] && !(ok = mbar_wait(smem_u32(b_qfull + 1), uses[1] & 1u, lim, kSiteQFull)))
                    break;
                if (m.active(1, m.lo)) s_step(m, 1, sk, m.lo);
                mma_commit(smem_u32(b_kvempty + sk));
                for (int j = m.lo; ok && j <= m.hi; ++j) {
                    uint32_t sv = 0;
                    if (!(ok = acquire(sv))) break;
                    if (m.active(0, j) && !(ok = pv_step(m, 0, sv, j))) break;
                    const bool next = j + 1 <= m.hi;
                    uint32_t sk2 = 0;
                    if (next) {
                        if (!(ok = acquire(sk2))) break;
                        if (m.active(0, j + 1)) s_step(m, 0, sk2, j + 1);
                    }
                    if (m.active(1, j) && !(ok = pv_step(m, 1, sv, j))) break;
                    mma_commit(smem_u32(b_kvempty + sv));
                    if (next) {
                        if (m.active(1, j + 1)) s_step(m, 1, sk2, j + 1);
                        mma_commit(smem_u32(b_kvempty + sk2));
                    }
                }
                for (int g = 0; g < 2; ++g)
                    if (m.valid[g]) ++uses[g];
            }
            // Drain: every tensor-core operation issued above has finished before teardown.
            mma_commit(smem_u32(b_mdrain));
            mbar_wait(smem_u32(b_mdrain), 0, lim, kSiteDrain);
        }
        __syncwarp();
    } else {
        // ============================ softmax + epilogue ============================
        const int g = (warp - kSoftmaxWarp0) >> 2;   // query tile of this warpgroup
        // A warp reaches the TMEM lanes of its quarter, 32 (warp % 4) .. + 31: row r of the tile.
        const int r = ((warp & 3) << 5) + lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t colS = g == 0 ? C::COL_S0 : C::COL_S1;
        const uint32_t colO = g == 0 ? C::COL_O0 : C::COL_O1;
        const uint64_t c1x2 = f2_pack(p.c1, p.c1);
        const uint64_t nc2x2 = f2_pack(-p.c2, -p.c2);
        PolyConsts pc;
        pc.shift = f2_pack(12582912.0f, 12582912.0f);      // 1.5 * 2^23
        pc.nshift = f2_pack(-12582912.0f, -12582912.0f);
        pc.neg1 = f2_pack(-1.f, -1.f);
        pc.c3 = f2_pack(0.0551716685295105f, 0.0551716685295105f);
        pc.c2 = f2_pack(0.2426111251115799f, 0.2426111251115799f);
        pc.c1 = f2_pack(0.6932609677314758f, 0.6932609677314758f);
        pc.c0 = f2_pack(0.9999280571937561f, 0.9999280571937561f);
        uint32_t s_phase = 0, o_uses = 0;
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            const uint32_t slot = k & 1u;
            int it = 0;
            if (lane == 0) {
                ok = mbar_wait(smem_u32(b_itfull + slot), (k >> 1) & 1u, lim, kSiteItem);
                it = s_item[slot];
                mbar_arrive(smem_u32(b_itempty + slot));
            }
            ok = __all_sync(0xffffffffu, ok);
            it = __shfl_sync(0xffffffffu, it, 0);
            if (!ok || it < 0) break;
            const Item<D> m = decode_item<D>(p, it);
            if (!m.valid[g]) continue;
            const int qi = m.q0[g] + r;           // this thread's query position
            uint64_t l2[4], lr2[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) l2[a] = lr2[a] = 0ull;
            for (int j = m.lo_t[g]; j <= m.hi_t[g]; ++j) {
                const bool w = mbar_wait(smem_u32(b_sfull + g), s_phase, lim, kSiteSFull);
                ok = __all_sync(0xffffffffu, w);
                if (!ok) break;
                s_phase ^= 1u;
                tc_fence_after();
                const int k0 = j * C::BN;
                const bool need_mask = (k0 + C::BN - 1 > m.q0[g]) || (m.q0[g] + C::BM - 1 - k0 >= p.W);
                // S row in four 32-column quarters; quarter c+1 loads while quarter c is
                // processed.  P of two quarters packs into 32 words, written over S columns that
                // were already read.
                uint32_t sq[2][32];
                uint32_t pk[32];
                auto quarter = [&](const uint32_t (&sv)[32], int cbase, int pkbase) {
                    if (!need_mask) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int a = (e >> 1) & 3;
                            pk[pkbase + (e >> 1)] =
                                (a == 3) ? softmax_pair_poly(sv[e], sv[e + 1], c1x2, nc2x2, pc, l2[a], lr2[a])
                                         : softmax_pair_mufu(sv[e], sv[e + 1], c1x2, nc2x2, l2[a], lr2[a]);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int kv = k0 + cbase + e;
                            // masked scores become -inf in log2 units, so exp gives exactly 0
                            const uint32_t m0 = ((unsigned)(qi - kv) >= (unsigned)p.W) ? 0xff800000u : sv[e];
                            const uint32_t m1 = ((unsigned)(qi - kv - 1) >= (unsigned)p.W) ? 0xff800000u : sv[e + 1];
                            pk[pkbase + (e >> 1)] = softmax_pair_mufu(m0, m1, c1x2, nc2x2, l2[e >> 1 & 3], lr2[e >> 1 & 3]);
                        }
                    }
                };
                tmem_ld32(tmem + lane_base + colS + 0, sq[0]);
                tmem_ld_wait();
                tmem_ld32(tmem + lane_base + colS + 32, sq[1]);
                quarter(sq[0], 0, 0);
                tmem_ld_wait();
                tmem_ld32(tmem + lane_base + colS + 64, sq[0]);
                quarter(sq[1], 32, 16);
                tmem_st32(tmem + lane_base + colS + 0, pk);
                tmem_ld_wait();
                tmem_ld32(tmem + lane_base + colS + 96, sq[1]);
                quarter(sq[0], 64, 0);
                tmem_ld_wait();
                quarter(sq[1], 96, 16);
                tmem_st32(tmem + lane_base + colS + 32, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(smem_u32(b_pfull + g));
            }
            if (!ok) break;
            {
                const bool w = mbar_wait(smem_u32(b_ofull + g), o_uses & 1u, lim, kSiteOFull);
                ok = __all_sync(0xffffffffu, w);
            }
            if (!ok) break;
            tc_fence_after();
            float l = 0.f, lr = 0.f;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                float u0, u1, w0, w1;
                f2_unpack(l2[a], u0, u1);
                f2_unpack(lr2[a], w0, w1);
                l += u0 + u1;
                lr += w0 + w1;
            }
            const float inv_l = 1.0f / lr;
            const bool row_ok = qi < p.T;
            __nv_bfloat16* orow = p.out + (((long long)m.b * p.T + qi) * p.H + m.h) * D;
            // Read all of O, then release it to the next item, then convert and store.
            uint32_t ov[D / 32][32];
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tmem + lane_base + colO + cc * 32, ov[cc]);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(smem_u32(b_oempty + g));
            ++o_uses;
            if (row_ok) {
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t w16[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w16[e] = pack_bf16x2(__uint_as_float(ov[cc][2 * e]) * inv_l,
                                             __uint_as_float(ov[cc][2 * e + 1]) * inv_l);
                    uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(w16[4 * e], w16[4 * e + 1], w16[4 * e + 2], w16[4 * e + 3]);
                }
                if (p.lse != nullptr) p.lse[((long long)m.b * p.H + m.h) * p.T + qi] = p.m0 + logf(l);
            }
        }
    }

    // ---- teardown: all tensor-memory traffic of this CTA is finished before the free.
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace swa
