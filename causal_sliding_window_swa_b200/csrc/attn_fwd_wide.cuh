// attn_fwd_wide.cuh -- the windowed attention forward for D = 128 with 256-key score products.
//
// Same computation as attn_fwd.cuh ("Let's reproduce GPT-2 (124M)" notes, sections 3 and 19;
// intelliparadigm "GPT-2 for $73", section 3.2): out = softmax(qhat khat^T / sqrt(D) + mask) v' and
// lse over the keys 0 <= i - j < W of each query row, on the prologue's qhat / khat / v'.
//
// Why a second kernel.  On B200 one tcgen05.mma of shape M = 128, K = 16 costs about 157 cycles for
// any N up to 128 and about 187 cycles for N = 256 (measured), so a 128-key step of the first kernel
// (eight score products of N = 128 and eight PV products of N = D = 128) is bound at 16 x 157 = 2512
// cycles, and that kernel runs within 10% of it.  Here the score product takes 256 keys at once:
// per 256 keys, 8 x 187 cycles of score products plus 16 x 157 of PV products, 2004 cycles per 128
// keys.
//
// Work item: one 128-row query tile of one (b, h), as in the first kernel; its key band
// [q0 - W + 1, q0 + 127] is walked in blocks of two 128-key tiles starting at the band's first tile
// (the last block's second tile, when past the band, is neither loaded nor multiplied into O).
// Tensor memory (512 columns): S (256 fp32 columns, one block of scores) | P (128 columns, the
// block's probabilities as bf16 pairs) | O (128 fp32 columns).  Q stays in shared memory (SS score
// products: the measured MMA cost is the same as with Q in tensor memory), its buffer freed once the
// item's last score product is done.
// Shared memory: Q (32 KB) | a ring of four 32 KB slots | the output staging tile (32 KB) |
// barriers | row-sum exchange.  A K block takes two adjacent slots (always an even pair), laid out
// so that its 256 keys form one N = 256 operand: slot s holds feature chunk 0 of keys 0-127 and
// 128-255, slot s + 1 chunk 1 (the 128-byte swizzle chunks are 32 KB apart); a V tile takes one slot
// in the usual layout.  Per block the producer loads K of the next block (two slots) and the two V
// tiles of this one (two slots), so K blocks always start at an even slot.
// Pipeline: the score product of block b + 1 is issued as soon as the softmax warps have read S(b)
// into registers (s_free) and runs while they finish P(b); P(b) is written to tensor memory after
// the PV product of block b - 1 has read P(b - 1) (p_free).  The tensor pipe sees ... PV(b - 1),
// S(b + 1), PV(b), S(b + 2) ... back to back.
// Softmax, offset, rounding of P, the row-sum exchange and the TMA-store epilogue are those of the
// first kernel (see attn_fwd.cuh); each softmax thread takes 64 keys of a block (four threads per
// row), in four 16-key chunks.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "attn_fwd.cuh"
#include "ptx.cuh"

namespace swa {

struct WideCfg {
    static constexpr int D = 128;
    static constexpr int BM = 128;
    static constexpr int CHUNK_BYTES = 128 * 128;      // 128 rows x 128 B
    static constexpr int SLOT_BYTES = 128 * D * 2;     // 32 KB
    static constexpr int NS = 4;                       // ring slots
    static constexpr int SMEM_Q = SLOT_BYTES;
    static constexpr int SMEM_KV = NS * SLOT_BYTES;
    static constexpr int SMEM_OUT = SLOT_BYTES;
    static constexpr int SMEM_BAR = 512;
    static constexpr int SMEM_LX = 4 * 128 * 8;
    static constexpr int SMEM_TOTAL = SMEM_Q + SMEM_KV + SMEM_OUT + SMEM_BAR + SMEM_LX;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0;
    static constexpr uint32_t COL_P = 256;
    static constexpr uint32_t COL_O = 384;
    static constexpr int THREADS = 576;
    static constexpr int SOFTMAX_THREADS = 512;
};

enum : unsigned int { kSiteSFree = 20, kSitePFree = 21, kSiteRing = 22 };

template <bool DOC = false>
__global__ void __launch_bounds__(576, 1)
    attn_fwd_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                         const FwdParams p) {
    using C = WideCfg;
    constexpr int D = C::D;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0u) {   // uniform: every thread leaves before any barrier
        if (threadIdx.x == 0) record_error(kErrLayout, 0);
        return;
    }
    uint8_t* sQ = smem_raw;
    uint8_t* sKV = sQ + C::SMEM_Q;
    uint8_t* sOut = sKV + C::SMEM_KV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + C::SMEM_OUT);
    uint64_t* b_qfull = bars + 0;
    uint64_t* b_qempty = bars + 1;
    uint64_t* b_ofull = bars + 2;
    uint64_t* b_oempty = bars + 3;
    uint64_t* b_mdrain = bars + 4;
    uint64_t* b_lxa = bars + 5;
    uint64_t* b_lxb = bars + 6;
    uint64_t* b_itfull = bars + 7;               // [2]
    uint64_t* b_itempty = bars + 9;              // [2]
    uint64_t* b_ostaged = bars + 11;
    uint64_t* b_ofree = bars + 12;
    uint64_t* b_sfull = bars + 13;               // S(b) complete
    uint64_t* b_sfree = bars + 14;               // S(b) read by every softmax thread
    uint64_t* b_pfull = bars + 15;               // P(b) written by every softmax thread
    uint64_t* b_pfree = bars + 16;               // PV(b) done reading P(b)
    uint64_t* b_kvfull = bars + 17;              // [NS]
    uint64_t* b_kvempty = bars + 17 + C::NS;     // [NS]
    int* s_item = reinterpret_cast<int*>(bars + 17 + 2 * C::NS);   // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_item + 2);
    float2* s_lx = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(bars) + C::SMEM_BAR);   // [4][128]
    static_assert(17 + 2 * C::NS <= (C::SMEM_BAR - 16) / 8, "barrier area");

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
        mbar_init(smem_u32(b_lxa), 3 * 128);
        mbar_init(smem_u32(b_lxb), 128);
        mbar_init(smem_u32(b_ostaged), C::SOFTMAX_THREADS);
        mbar_init(smem_u32(b_ofree), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(b_itfull + i), 1);
            mbar_init(smem_u32(b_itempty + i), kItemConsumers);
        }
        mbar_init(smem_u32(b_sfull), 1);
        mbar_init(smem_u32(b_sfree), C::SOFTMAX_THREADS);
        mbar_init(smem_u32(b_pfull), C::SOFTMAX_THREADS);
        mbar_init(smem_u32(b_pfree), 1);
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
        tma_prefetch_desc(&tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = p.wait_limit_ns;
    // blocks of an item: pairs of 128-key tiles from the band's first tile
    auto n_blocks = [](const Item& m) { return (m.hi - m.lo + 2) >> 1; };

    if (warp == kProducerWarp) {
        // ========================= scheduler + TMA producer =========================
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t filled_phase[C::NS];
            bool filled[C::NS];
            for (int s = 0; s < C::NS; ++s) filled[s] = false, filled_phase[s] = 0;
            uint32_t q_uses = 0;
            bool ok = true;
            auto next = [&]() {
                if (++stage == (uint32_t)C::NS) {
                    stage = 0;
                    phase ^= 1u;
                }
            };
            // K of block b: two adjacent slots; slot s + c holds feature chunk c of both tiles.
            auto load_k = [&](const Item& m, int b) -> bool {
                if ((stage & 1u) != 0u) {        // cannot happen: K blocks start at even slots
                    record_error(kErrLayout, kSiteRing);
                    return false;
                }
                const bool live1 = m.lo + 2 * b + 1 <= m.hi;
                for (int c = 0; c < 2; ++c) {
                    if (!mbar_wait(smem_u32(b_kvempty + stage), phase ^ 1u, lim, kSiteKvEmpty)) return false;
                    const uint32_t fb = smem_u32(b_kvfull + stage);
                    mbar_arrive_expect_tx(fb, (uint32_t)(live1 ? 2 * C::CHUNK_BYTES : C::CHUNK_BYTES));
                    for (int h = 0; h < (live1 ? 2 : 1); ++h)
                        tma_load_4d(smem_u32(sKV + stage * C::SLOT_BYTES + h * C::CHUNK_BYTES), &tm_k, fb, c * 64,
                                    m.h / p.G, (m.lo + 2 * b + h) * 128, m.b);
                    filled[stage] = true;
                    filled_phase[stage] = phase;
                    next();
                }
                return true;
            };
            // V tile h of block b: one slot, chunk c at c * 16 KB; a tile past the band is skipped
            // (its slot completes with no bytes).
            auto load_v = [&](const Item& m, int b, int h) -> bool {
                if (!mbar_wait(smem_u32(b_kvempty + stage), phase ^ 1u, lim, kSiteKvEmpty)) return false;
                const uint32_t fb = smem_u32(b_kvfull + stage);
                if (m.lo + 2 * b + h <= m.hi) {
                    mbar_arrive_expect_tx(fb, (uint32_t)C::SLOT_BYTES);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(smem_u32(sKV + stage * C::SLOT_BYTES + c * C::CHUNK_BYTES), &tm_v, fb, c * 64,
                                    m.h / p.G, (m.lo + 2 * b + h) * 128, m.b);
                } else {
                    mbar_arrive(fb);
                }
                filled[stage] = true;
                filled_phase[stage] = phase;
                next();
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
                const Item m = decode_item(p, it);
                const int nb = n_blocks(m);
                for (int ch = 0; ch < 2; ++ch) tma_prefetch_4d(&tm_q, ch * 64, m.h, m.q0, m.b);
                if (q_uses > 0 && !(ok = mbar_wait(smem_u32(b_qempty), (q_uses - 1) & 1u, lim, kSiteQEmpty)))
                    break;
                {
                    const uint32_t qb = smem_u32(b_qfull);
                    mbar_arrive_expect_tx(qb, (uint32_t)C::SLOT_BYTES);
                    for (int ch = 0; ch < 2; ++ch)
                        tma_load_4d(smem_u32(sQ + ch * C::CHUNK_BYTES), &tm_q, qb, ch * 64, m.h, m.q0, m.b);
                    ++q_uses;
                }
                // The MMA thread's order: K(0), then K(b + 1), V(b, 0), V(b, 1) for each block b.
                ok = load_k(m, 0);
                for (int b = 0; ok && b < nb; ++b)
                    ok = (b + 1 >= nb || load_k(m, b + 1)) && load_v(m, b, 0) && load_v(m, b, 1);
            }
            if (ok && atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
                p.sched[0] = 0;
                p.sched[1] = 0;
            }
            if (q_uses > 0) mbar_wait(smem_u32(b_qfull), (q_uses - 1) & 1u, lim, kSiteDrain);
            for (int s = 0; s < C::NS; ++s)
                if (filled[s]) mbar_wait(smem_u32(b_kvfull + s), filled_phase[s], lim, kSiteDrain);
        }
    } else if (warp == kMmaWarp) {
        // ============================== MMA issuer ==============================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 256, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dkv = smem_desc_sw128(smem_u32(sKV), 16, 1024);
            const uint64_t dv = smem_desc_sw128(smem_u32(sKV), C::CHUNK_BYTES, 1024);
            const uint32_t d_s = tmem + C::COL_S, d_o = tmem + C::COL_O, a_p = tmem + C::COL_P;
            uint32_t stage = 0, phase = 0;
            uint32_t bs = 0;     // score blocks issued (all items)
            uint32_t bp = 0;     // PV blocks issued
            uint32_t uses = 0;   // items done
            auto acquire = [&](uint32_t& s) -> bool {
                s = stage;
                const bool r = mbar_wait(smem_u32(b_kvfull + stage), phase, lim, kSiteKvFull);
                if (++stage == (uint32_t)C::NS) {
                    stage = 0;
                    phase ^= 1u;
                }
                return r;
            };
            // S(b) = Q K_b^T: M = 128, N = 256 keys, K = D in 16-steps.  Q (A) K-major from shared
            // memory; K (B) K-major across the slot pair (chunk c in slot s + c).  S is overwritten
            // only after the softmax warps have read the previous block (s_free).
            auto s_step = [&](bool last_of_item) -> bool {
                if (bs > 0 && !mbar_wait(smem_u32(b_sfree), (bs - 1) & 1u, lim, kSiteSFree)) return false;
                uint32_t s0 = 0, s1 = 0;
                if (!acquire(s0) || !acquire(s1)) return false;
                tc_fence_after();
                const uint64_t db = dkv + (uint64_t)((s0 * C::SLOT_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::SLOT_BYTES + (kk & 3) * 32) >> 4;
                    const uint32_t qoff = ((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4;
                    mma_ss(d_s, dq + qoff, db + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(b_sfull));
                mma_commit(smem_u32(b_kvempty + s0));
                mma_commit(smem_u32(b_kvempty + s1));
                if (last_of_item) mma_commit(smem_u32(b_qempty));
                ++bs;
                return true;
            };
            // O += P(b) V(b): M = 128, N = D, K = 256 keys in 16-steps; P from tensor memory (key g of
            // the block at column g / 2), V MN-major, tile h in its own slot.
            auto pv_step = [&](const Item& m, int b, bool first, bool last) -> bool {
                if (!mbar_wait(smem_u32(b_pfull), bp & 1u, lim, kSitePFull)) return false;
                if (first && uses > 0 && !mbar_wait(smem_u32(b_oempty), (uses - 1) & 1u, lim, kSiteOEmpty))
                    return false;
                tc_fence_after();
                for (int h = 0; h < 2; ++h) {
                    uint32_t sv = 0;
                    if (!acquire(sv)) return false;
                    if (m.lo + 2 * b + h <= m.hi) {
                        const uint64_t db = dv + (uint64_t)((sv * C::SLOT_BYTES) >> 4);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ts(d_o, a_p + 64u * (uint32_t)h + 8u * (uint32_t)kk,
                                   db + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                                   (!first || h > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(smem_u32(b_kvempty + sv));
                }
                mma_commit(smem_u32(b_pfree));
                if (last) mma_commit(smem_u32(b_ofull));
                ++bp;
                return true;
            };

            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                const uint32_t slot = k & 1u;
                if (!(ok = mbar_wait(smem_u32(b_itfull + slot), (k >> 1) & 1u, lim, kSiteItem))) break;
                const int it = s_item[slot];
                mbar_arrive(smem_u32(b_itempty + slot));
                if (it < 0) break;
                const Item m = decode_item(p, it);
                const int nb = n_blocks(m);
                if (!(ok = mbar_wait(smem_u32(b_qfull), uses & 1u, lim, kSiteQFull))) break;
                ok = s_step(nb == 1);
                for (int b = 0; ok && b < nb; ++b)
                    ok = (b + 1 >= nb || s_step(b + 2 == nb)) && pv_step(m, b, b == 0, b + 1 == nb);
                ++uses;
            }
            mma_commit(smem_u32(b_mdrain));
            mbar_wait(smem_u32(b_mdrain), 0, lim, kSiteDrain);
        }
        __syncwarp();
    } else {
        // ============================ softmax + epilogue ============================
        const int cq = (warp - kSoftmaxWarp0) >> 2;   // key quarter of a block / output column quarter
        const int r = ((warp & 3) << 5) + lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint64_t c1x2 = f2_pack(p.c1, p.c1);
        const uint64_t nc2x2 = f2_pack(-p.c2, -p.c2);
        PolyConsts pc;
        pc.shift = f2_pack(12582912.0f, 12582912.0f);      // 1.5 * 2^23
        pc.c3 = f2_pack(0.0551716685295105f, 0.0551716685295105f);
        pc.c2 = f2_pack(0.2426111251115799f, 0.2426111251115799f);
        pc.c1 = f2_pack(0.6932609677314758f, 0.6932609677314758f);
        pc.c0 = f2_pack(0.9999280571937561f, 0.9999280571937561f);
        uint32_t blk = 0, o_uses = 0;
        const bool is_store = (warp == kSoftmaxWarp0 && lane == 0);
        bool ok = true;

        auto fetch = [&](uint32_t kk) -> int {
            const uint32_t slot = kk & 1u;
            int v = 0;
            bool w = true;
            if (lane == 0) {
                w = mbar_wait(smem_u32(b_itfull + slot), (kk >> 1) & 1u, lim, kSiteItem);
                v = s_item[slot];
                mbar_arrive(smem_u32(b_itempty + slot));
            }
            const bool all = __all_sync(0xffffffffu, w);
            ok = ok && all;
            v = __shfl_sync(0xffffffffu, v, 0);
            return ok ? v : -1;
        };

        uint32_t k = 0;
        int it = fetch(0);
        while (ok && it >= 0) {
            const Item m = decode_item(p, it);
            const int nb = n_blocks(m);
            const int qi = m.q0 + r;
            int ds = 0, ds_w = 0;
            if constexpr (DOC) {
                ds = __ldg(p.dstart + (long long)m.b * p.T + min(qi, p.T - 1));
                ds_w = __reduce_max_sync(0xffffffffu, ds);
            }
            uint64_t l2[4], lr2[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) l2[a] = lr2[a] = 0ull;
            for (int b = 0; b < nb; ++b, ++blk) {
                {
                    const bool w = mbar_wait(smem_u32(b_sfull), blk & 1u, lim, kSiteSFull);
                    ok = __all_sync(0xffffffffu, w);
                }
                if (!ok) break;
                tc_fence_after();
                const int kt = (m.lo + 2 * b) * 128 + 64 * cq;          // first key of this thread
                const bool dead = m.lo + 2 * b + (cq >> 1) > m.hi;      // this quarter's tile is past the band
                uint32_t pw[32];
                // 16 keys (scores sv) -> 8 bf16 pairs at pw[pbase..]
                auto chunk = [&](const uint32_t (&sv)[16], int c) {
                    const int kc = kt + 16 * c;
                    const bool need_mask = (kc + 15 > m.q0) || (m.q0 + C::BM - 1 - kc >= p.W) || (DOC && kc < ds_w);
                    if (!need_mask) {
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const int a = (e >> 1) & 3;
                            pw[8 * c + (e >> 1)] =
                                ((kPolyPairMask >> (e >> 1)) & 1u)
                                    ? softmax_pair_poly(sv[e], sv[e + 1], c1x2, nc2x2, pc, l2[a], lr2[a])
                                    : softmax_pair_mufu(sv[e], sv[e + 1], c1x2, nc2x2, l2[a], lr2[a]);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const int kv = kc + e;
                            const uint32_t m0 = ((unsigned)(qi - kv) >= (unsigned)p.W || (DOC && kv < ds))
                                                    ? 0xff800000u : sv[e];
                            const uint32_t m1 = ((unsigned)(qi - kv - 1) >= (unsigned)p.W || (DOC && kv + 1 < ds))
                                                    ? 0xff800000u : sv[e + 1];
                            pw[8 * c + (e >> 1)] = softmax_pair_mufu(m0, m1, c1x2, nc2x2, l2[e >> 1 & 3], lr2[e >> 1 & 3]);
                        }
                    }
                };
                const uint32_t colS = tmem + lane_base + C::COL_S + 64u * (uint32_t)cq;
                if (!dead) {
                    uint32_t sa[16], sb[16];
                    tmem_ld16(colS + 0, sa);
                    tmem_ld16(colS + 16, sb);
                    tmem_ld_wait();
                    chunk(sa, 0);
                    chunk(sb, 1);
                    tmem_ld16(colS + 32, sa);
                    tmem_ld16(colS + 48, sb);
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(smem_u32(b_sfree));      // S may now be overwritten
                    chunk(sa, 2);
                    chunk(sb, 3);
                } else {
                    // keys past the band: probability 0, scores never read
#pragma unroll
                    for (int e = 0; e < 32; ++e) pw[e] = 0u;
                    tc_fence_before();
                    mbar_arrive(smem_u32(b_sfree));
                }
                // P(b) replaces P(b - 1) once the PV product of the previous block has read it.
                if (blk > 0) {
                    const bool w = mbar_wait(smem_u32(b_pfree), (blk - 1) & 1u, lim, kSitePFree);
                    ok = __all_sync(0xffffffffu, w);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t colP = tmem + lane_base + C::COL_P + 32u * (uint32_t)cq;
                tmem_st16(colP, *reinterpret_cast<const uint32_t(*)[16]>(pw));
                tmem_st16(colP + 16, *reinterpret_cast<const uint32_t(*)[16]>(pw + 16));
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(smem_u32(b_pfull));
            }
            if (!ok) break;
            float l = 0.f, lr = 0.f;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                float u0, u1, w0, w1;
                f2_unpack(l2[a], u0, u1);
                f2_unpack(lr2[a], w0, w1);
                l += u0 + u1;
                lr += w0 + w1;
            }
            ++k;
            const int it_next = fetch(k);
            if (!ok) break;
            {
                const bool w = mbar_wait(smem_u32(b_ofull), o_uses & 1u, lim, kSiteOFull);
                ok = __all_sync(0xffffffffu, w);
            }
            if (!ok) break;
            tc_fence_after();
            constexpr int OQ = D / 4;             // 32 output columns per thread
            uint32_t ov[OQ];
            tmem_ld16(tmem + lane_base + C::COL_O + (uint32_t)(OQ * cq), *reinterpret_cast<uint32_t(*)[16]>(ov));
            tmem_ld16(tmem + lane_base + C::COL_O + (uint32_t)(OQ * cq) + 16u,
                      *reinterpret_cast<uint32_t(*)[16]>(ov + 16));
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(smem_u32(b_oempty));
            ++o_uses;
            const uint32_t xpar = (o_uses - 1u) & 1u;
            if (cq != 0) {
                s_lx[cq * 128 + r] = make_float2(l, lr);
                mbar_arrive(smem_u32(b_lxa));
                ok = mbar_wait(smem_u32(b_lxb), xpar, lim, kSiteRowSum);
                const float2 t = s_lx[r];
                l = t.x;
                lr = t.y;
            } else {
                ok = mbar_wait(smem_u32(b_lxa), xpar, lim, kSiteRowSum);
#pragma unroll
                for (int c = 1; c < 4; ++c) {
                    const float2 t = s_lx[c * 128 + r];
                    l += t.x;
                    lr += t.y;
                }
                s_lx[r] = make_float2(l, lr);
                mbar_arrive(smem_u32(b_lxb));
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const float inv_l = 1.0f / lr;
            const uint32_t e_idx = o_uses - 1u;
            if (e_idx > 0) {
                if (is_store) {
                    bulk_wait_read_all();
                    mbar_arrive(smem_u32(b_ofree));
                }
                ok = mbar_wait(smem_u32(b_ofree), (e_idx - 1u) & 1u, lim, kSiteOStage);
            }
            {
                uint32_t w16[OQ / 2];
#pragma unroll
                for (int e = 0; e < OQ / 2; ++e)
                    w16[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l, __uint_as_float(ov[2 * e + 1]) * inv_l);
                const int col0 = OQ * cq;
                uint8_t* rowp = sOut + (col0 >> 6) * C::CHUNK_BYTES + r * 128;
                const int u0 = (col0 & 63) >> 3;
#pragma unroll
                for (int e = 0; e < OQ / 8; ++e)
                    *reinterpret_cast<uint4*>(rowp + (((u0 + e) ^ (r & 7)) << 4)) =
                        make_uint4(w16[4 * e], w16[4 * e + 1], w16[4 * e + 2], w16[4 * e + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(b_ostaged));
            if (is_store) {
                if (mbar_wait(smem_u32(b_ostaged), e_idx & 1u, lim, kSiteOStage)) {
                    for (int ch = 0; ch < 2; ++ch)
                        tma_store_4d(&tm_o, smem_u32(sOut + ch * C::CHUNK_BYTES), ch * 64, m.h, m.q0, m.b);
                    bulk_commit_group();
                } else {
                    ok = false;
                }
            }
            if (qi < p.T && cq == 0 && p.lse != nullptr)
                p.lse[((long long)m.b * p.H + m.h) * p.T + qi] = p.m0 + logf(l);
            ok = __all_sync(0xffffffffu, ok);
            it = it_next;
        }
    }

    if (warp == kSoftmaxWarp0 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace swa
