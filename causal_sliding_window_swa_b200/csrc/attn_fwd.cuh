// attn_fwd.cuh -- causal sliding-window attention forward on the sm_100a tensor cores.
//
// What it computes ("Let's reproduce GPT-2 (124M)" notes, section 3 and section 19;
// intelliparadigm "GPT-2 for $73", section 3.2):
//   out[b,i,h,:] = sum_{j in J_i} softmax_j(qhat_i . khat_j / sqrt(D)) v'_j,
//   J_i = { j : 0 <= i - j < W },  lse[b,h,i] = ln sum_{j in J_i} exp(qhat_i . khat_j / sqrt(D)),
// on the RMS-normalised, rotated qhat/khat and the gated v' that the prologue wrote.
//
// One CTA owns two adjacent 128-row query tiles of one (b, h) and walks the 128-row key/value
// tiles that intersect their window band [q0 - W + 1, q0 + 255]; tiles outside the band are
// never loaded.  Warp roles (320 threads):
//   warps 0-3  softmax/epilogue for query tile 0 (thread r owns row r: TMEM lane r)
//   warps 4-7  softmax/epilogue for query tile 1
//   warp  8    TMA producer: Q tiles once, then K_j, V_j through an NS-stage mbarrier ring
//   warp  9    TMEM allocator and the single thread that issues tcgen05.mma
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
// One exponential in four is evaluated by a polynomial on the FMA pipe to offload the MUFU unit,
// which otherwise limits the softmax at the rate of the tensor core.
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
    static constexpr int NS = (D == 128) ? 4 : 8;      // K/V ring depth
    static constexpr int SMEM_Q = 2 * TILE_BYTES;
    static constexpr int SMEM_KV = NS * TILE_BYTES;
    static constexpr int SMEM_BAR = 256;
    static constexpr int SMEM_TOTAL = 1024 /*alignment slack*/ + SMEM_Q + SMEM_KV + SMEM_BAR;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
    static constexpr int THREADS = 320;
};

struct FwdParams {
    int B, T, H;
    int W;                 // effective window, 1..T
    int n_pairs;           // ceil(ceil(T/128)/2)
    float c1;              // log2(e) / sqrt(D): raw score -> log2 units
    float c2;              // M0 * log2(e)
    float m0;              // M0 (natural-log units), added back into the LSE
    __nv_bfloat16* out;    // (B,T,H,D)
    float* lse;            // (B,H,T) or null
    unsigned long long wait_limit_ns;
};

// Wait sites recorded in the status word on timeout.
enum : unsigned int {
    kSiteQFull = 1, kSiteKvEmpty = 2, kSiteKvFull = 3, kSiteSFull = 4, kSitePFull = 5,
    kSiteOFull = 6, kSiteDrain = 7
};

template <int D>
__global__ void __maxnreg__(200)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;                          // 2 tiles
    uint8_t* sKV = smem + C::SMEM_Q;             // NS tiles
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_Q + C::SMEM_KV);
    // barrier slots
    uint64_t* b_qfull = bars + 0;
    uint64_t* b_kvfull = bars + 1;               // [NS]
    uint64_t* b_kvempty = bars + 1 + C::NS;      // [NS]
    uint64_t* b_sfull = bars + 1 + 2 * C::NS;    // [2]
    uint64_t* b_pfull = b_sfull + 2;             // [2]
    uint64_t* b_ofull = b_pfull + 2;             // [2]
    uint64_t* b_mdrain = b_ofull + 2;            // MMA thread's final drain
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(b_mdrain + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work item: query-tile pair (heaviest first), head, batch row
    const int pair = p.n_pairs - 1 - (int)blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int T = p.T, W = p.W;
    int q0[2], lo_t[2], hi_t[2];
    bool valid[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        q0[g] = (2 * pair + g) * C::BM;
        valid[g] = q0[g] < T;
        const int first_key = max(0, q0[g] - W + 1);
        const int last_key = min(q0[g] + C::BM - 1, T - 1);
        lo_t[g] = first_key / C::BN;
        hi_t[g] = last_key / C::BN;
    }
    const int lo = lo_t[0];
    const int hi = valid[1] ? hi_t[1] : hi_t[0];
    auto active = [&](int g, int j) { return valid[g] && j >= lo_t[g] && j <= hi_t[g]; };

    // ---- barrier init (one thread), TMEM allocation (warp 9)
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(b_qfull), 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(smem_u32(b_kvfull + s), 1);
            mbar_init(smem_u32(b_kvempty + s), 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(smem_u32(b_sfull + g), 1);
            mbar_init(smem_u32(b_pfull + g), 128);
            mbar_init(smem_u32(b_ofull + g), 1);
        }
        mbar_init(smem_u32(b_mdrain), 1);
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = p.wait_limit_ns;

    if (warp == 8) {
        // ============================== TMA producer ==============================
        if (lane == 0) {
            const uint32_t qbar = smem_u32(b_qfull);
            mbar_arrive_expect_tx(qbar, (valid[1] ? 2u : 1u) * (uint32_t)C::TILE_BYTES);
            for (int g = 0; g < 2; ++g) {
                if (!valid[g]) continue;
                for (int ch = 0; ch < C::NCHUNK; ++ch)
                    tma_load_4d(smem_u32(sQ + g * C::TILE_BYTES + ch * C::CHUNK_BYTES), &tm_q,
                                qbar, ch * 64, h, q0[g], b);
            }
            uint32_t stage = 0, phase = 0;
            uint32_t filled_phase[C::NS];
            bool filled[C::NS];
            for (int s = 0; s < C::NS; ++s) filled[s] = false, filled_phase[s] = 0;
            bool ok = true;
            for (int j = lo; ok && j <= hi; ++j) {
                for (int which = 0; which < 2; ++which) {
                    if (!mbar_wait(smem_u32(b_kvempty + stage), phase ^ 1u, lim, kSiteKvEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(b_kvfull + stage);
                    mbar_arrive_expect_tx(fb, (uint32_t)C::TILE_BYTES);
                    const CUtensorMap* tm = which == 0 ? &tm_k : &tm_v;
                    for (int ch = 0; ch < C::NCHUNK; ++ch)
                        tma_load_4d(smem_u32(sKV + stage * C::TILE_BYTES + ch * C::CHUNK_BYTES),
                                    tm, fb, ch * 64, h, j * C::BN, b);
                    filled[stage] = true;
                    filled_phase[stage] = phase;
                    if (++stage == (uint32_t)C::NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Drain: every copy this thread started has landed before the CTA may exit.
            mbar_wait(qbar, 0, lim, kSiteDrain);
            for (int s = 0; s < C::NS; ++s)
                if (filled[s]) mbar_wait(smem_u32(b_kvfull + s), filled_phase[s], lim, kSiteDrain);
        }
    } else if (warp == 9) {
        // ============================== MMA issuer ==============================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, C::BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            const uint32_t sQ_addr = smem_u32(sQ);
            const uint32_t sKV_addr = smem_u32(sKV);
            uint32_t stage = 0, phase = 0;
            uint32_t p_phase[2] = {0u, 0u};
            auto acquire = [&](uint32_t& s) -> bool {
                s = stage;
                const bool r = mbar_wait(smem_u32(b_kvfull + stage), phase, lim, kSiteKvFull);
                if (++stage == (uint32_t)C::NS) {
                    stage = 0;
                    phase ^= 1u;
                }
                return r;
            };
            // S_g = Q_g K^T : M=128, N=BN, K=D in steps of 16 (32 bytes inside a swizzle chunk).
            auto issue_s = [&](int g, uint32_t sk) {
                const uint32_t a0 = sQ_addr + g * C::TILE_BYTES;
                const uint32_t b0 = sKV_addr + sk * C::TILE_BYTES;
                const uint32_t d = tmem + (g == 0 ? C::COL_S0 : C::COL_S1);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32;
                    mma_ss(d, smem_desc_sw128(a0 + off, 16, 1024), smem_desc_sw128(b0 + off, 16, 1024),
                           idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O_g += P_g V : M=128, N=D, K=BN in steps of 16 key rows.  P from tensor memory
            // (8 columns of packed bf16 pairs per step), V MN-major from shared memory.
            auto issue_pv = [&](int g, uint32_t sv, bool acc) {
                const uint32_t pa = tmem + (g == 0 ? C::COL_S0 : C::COL_S1);
                const uint32_t b0 = sKV_addr + sv * C::TILE_BYTES;
                const uint32_t d = tmem + (g == 0 ? C::COL_O0 : C::COL_O1);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    mma_ts(d, pa + kk * 8, smem_desc_sw128(b0 + kk * 16 * 128, C::CHUNK_BYTES, 1024),
                           idesc_pv, (acc || kk > 0) ? 1u : 0u);
                }
            };

            bool ok = mbar_wait(smem_u32(b_qfull), 0, lim, kSiteQFull);
            uint32_t sk = 0;
            if (ok) ok = acquire(sk);
            if (ok) {
                tc_fence_after();
                for (int g = 0; g < 2; ++g)
                    if (active(g, lo)) {
                        issue_s(g, sk);
                        mma_commit(smem_u32(b_sfull + g));
                    }
                mma_commit(smem_u32(b_kvempty + sk));
            }
            for (int j = lo; ok && j <= hi; ++j) {
                uint32_t sv = 0;
                if (!(ok = acquire(sv))) break;
                tc_fence_after();
                if (active(0, j)) {
                    if (!(ok = mbar_wait(smem_u32(b_pfull + 0), p_phase[0], lim, kSitePFull))) break;
                    p_phase[0] ^= 1u;
                    tc_fence_after();
                    issue_pv(0, sv, j > lo_t[0]);
                    if (j == hi_t[0]) mma_commit(smem_u32(b_ofull + 0));
                }
                const bool next = j + 1 <= hi;
                uint32_t sk2 = 0;
                if (next) {
                    if (!(ok = acquire(sk2))) break;
                    tc_fence_after();
                    if (active(0, j + 1)) {
                        issue_s(0, sk2);
                        mma_commit(smem_u32(b_sfull + 0));
                    }
                }
                if (active(1, j)) {
                    if (!(ok = mbar_wait(smem_u32(b_pfull + 1), p_phase[1], lim, kSitePFull))) break;
                    p_phase[1] ^= 1u;
                    tc_fence_after();
                    issue_pv(1, sv, j > lo_t[1]);
                    if (j == hi_t[1]) mma_commit(smem_u32(b_ofull + 1));
                }
                mma_commit(smem_u32(b_kvempty + sv));
                if (next) {
                    if (active(1, j + 1)) {
                        issue_s(1, sk2);
                        mma_commit(smem_u32(b_sfull + 1));
                    }
                    mma_commit(smem_u32(b_kvempty + sk2));
                }
            }
            // Drain: every tensor-core operation issued above has finished before teardown.
            mma_commit(smem_u32(b_mdrain));
            mbar_wait(smem_u32(b_mdrain), 0, lim, kSiteDrain);
        }
        __syncwarp();
    } else {
        // ============================ softmax + epilogue ============================
        const int g = warp >> 2;                  // query tile of this warpgroup
        const int r = ((warp & 3) << 5) + lane;   // row within the tile == TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t colS = g == 0 ? C::COL_S0 : C::COL_S1;
        const uint32_t colO = g == 0 ? C::COL_O0 : C::COL_O1;
        const int qi = q0[g] + r;                 // this thread's query position
        // Row sums, kept in 4 independent fp32 pairs each so the adds do not form one chain:
        // l  = sum of exp(s - M0) (for the LSE), lr = sum of the bf16 P the PV product uses
        // (the normaliser of the output).
        uint64_t l2[4], lr2[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) l2[a] = lr2[a] = 0ull;
        bool ok = true;
        if (valid[g]) {
            const uint64_t c1x2 = f2_pack(p.c1, p.c1);
            const uint64_t nc2x2 = f2_pack(-p.c2, -p.c2);
            uint32_t s_phase = 0;
            for (int j = lo_t[g]; j <= hi_t[g]; ++j) {
                bool w = mbar_wait(smem_u32(b_sfull + g), s_phase, lim, kSiteSFull);
                ok = __all_sync(0xffffffffu, w);
                if (!ok) break;
                s_phase ^= 1u;
                tc_fence_after();
                const int k0 = j * C::BN;
                const bool need_mask = (k0 + C::BN - 1 > q0[g]) || (q0[g] + C::BM - 1 - k0 >= W);
                // S row in four 32-column quarters; quarter c+1 loads while quarter c is processed.
                // P of two quarters (64 columns) packs into 32 words, written over S columns
                // that were already read.
                uint32_t sq[2][32];
                uint32_t pk[32];
                auto softmax_quarter = [&](const uint32_t (&sv)[32], int cbase, int pkbase) {
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])),
                                                  c1x2, nc2x2);
                        float p0, p1;
                        if (((e >> 1) & 3) == 3) {
                            // one pair in four on the FMA pipe, the rest on MUFU
                            f2_unpack(exp2_poly_x2(x), p0, p1);
                        } else {
                            float x0, x1;
                            f2_unpack(x, x0, x1);
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                        }
                        if (need_mask) {
                            const int kv = k0 + cbase + e;
                            if ((unsigned)(qi - kv) >= (unsigned)W) p0 = 0.f;
                            if ((unsigned)(qi - kv - 1) >= (unsigned)W) p1 = 0.f;
                        }
                        const int a = (e >> 1) & 3;
                        l2[a] = f2_add(l2[a], f2_pack(p0, p1));
                        // bf16 by truncation; the normaliser sums exactly these values
                        lr2[a] = f2_add(lr2[a], f2_pack(__uint_as_float(__float_as_uint(p0) & 0xffff0000u),
                                                        __uint_as_float(__float_as_uint(p1) & 0xffff0000u)));
                        pk[pkbase + (e >> 1)] = pack_bf16x2_trunc(p0, p1);
                    }
                };
                tmem_ld32(tmem + lane_base + colS + 0, sq[0]);
                tmem_ld_wait();
                tmem_ld32(tmem + lane_base + colS + 32, sq[1]);
                softmax_quarter(sq[0], 0, 0);
                tmem_ld_wait();
                tmem_ld32(tmem + lane_base + colS + 64, sq[0]);
                softmax_quarter(sq[1], 32, 16);
                tmem_st32(tmem + lane_base + colS + 0, pk);
                tmem_ld_wait();
                tmem_ld32(tmem + lane_base + colS + 96, sq[1]);
                softmax_quarter(sq[0], 64, 0);
                tmem_ld_wait();
                softmax_quarter(sq[1], 96, 16);
                tmem_st32(tmem + lane_base + colS + 32, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(smem_u32(b_pfull + g));
            }
            if (ok) {
                bool w = mbar_wait(smem_u32(b_ofull + g), 0, lim, kSiteOFull);
                ok = __all_sync(0xffffffffu, w);
            }
            if (ok) {
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
                const bool row_ok = qi < T;
                __nv_bfloat16* orow = p.out + (((long long)b * T + qi) * p.H + h) * D;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t ov[32];
                    tmem_ld32(tmem + lane_base + colO + cc * 32, ov);
                    tmem_ld_wait();
                    if (row_ok) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l,
                                                __uint_as_float(ov[2 * e + 1]) * inv_l);
                        uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                    }
                }
                if (row_ok && p.lse != nullptr)
                    p.lse[((long long)b * p.H + h) * T + qi] = p.m0 + logf(l);
            }
        }
    }

    // ---- teardown: all tensor-memory traffic of this CTA is finished before the free.
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace swa
