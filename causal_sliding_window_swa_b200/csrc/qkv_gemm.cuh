// qkv_gemm.cuh -- the q, k, v projection of the layer input fused with the prologue, on the
// sm_100a tensor cores.
//
// What it computes (the bias-free q, k, v maps of "Let's reproduce GPT-2 (124M)" notes, section 3,
// and intelliparadigm "GPT-2 for $73", section 2; then RoPE -> RMS on q and k, section 2.2 there,
// and the gated value embedding of the PaperWeekly repost, "Value Embeddings" paragraph):
//   y[t, n] = sum_c x[t, c] Wqkv[n, c]                 (x (B*T, C), Wqkv [(H + 2 Hkv) D, C])
//   qhat = rms(rope(y[:, q head])), khat = rms(rope(y[:, k head])),
//   v'   = y[:, v head] + g ve,  g = 2 sigmoid(x[t, :32] . Wg[:, h]) (precomputed by gate_kernel),
// written as bf16 (round to nearest) in the (B, T, heads, D) layouts the attention kernel reads.
// The projection stays in fp32 (tensor-memory accumulator) through the epilogue: q, k, v are
// never rounded or written to global memory.
//
// Tiles: 128 tokens x BN output features (BN = 256 when the q, k and v widths are multiples of
// 256, else 128), K = C in chunks of 64 (one 128-byte swizzle atom), an NS-stage TMA ring for the
// x and Wqkv chunks.  Persistent CTAs walk the tiles in the order tile = blockIdx.x + k gridDim.x,
// token block major, so CTAs running at the same time share x rows in L2 (Wqkv, a few MB, stays
// in L2).  Two accumulator buffers in tensor memory let the epilogue of one tile overlap the
// products of the next.
// Warp roles: warp 0 issues the tensor-core products, warp 1 is the TMA producer, warps
// 2 .. 2 + 4 BN / 128 - 1 run the epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (one
// token each) and the 128 accumulator columns 128 ((w - 2) / 4) .. + 127 of them, which hold one
// head (D = 128) or two (D = 64).  A thread therefore owns whole head rows: the RMS sum and the
// RoPE pairs (i, i + D/2) never leave it.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace swa {

// 2-D tiled load of one box into shared memory, completing its bytes on the mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

template <int BN>
struct QkvCfg {
    static constexpr int BM = 128;                       // tokens per tile (MMA M)
    static constexpr int BK = 64;                        // contraction chunk: 128 bytes of bf16
    static constexpr int A_BYTES = BM * BK * 2;          // 16 KB
    static constexpr int B_BYTES = BN * BK * 2;          // 16 or 32 KB
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int NS = (BN == 256) ? 4 : 6;
    static constexpr int SMEM_BAR = 256;
    static constexpr int SMEM_TOTAL = NS * STAGE_BYTES + SMEM_BAR;
    static constexpr int EPI_WARPS = 4 * (BN / 128);
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr uint32_t TMEM_COLS = 2 * BN;        // two accumulator buffers
    static_assert(SMEM_TOTAL <= 227 * 1024, "shared memory per CTA");
};

struct QkvParams {
    int M;                 // B * T tokens
    int T;
    int C;
    int H, Hkv;
    int n_ntiles;          // (H + 2 Hkv) D / BN
    int n_tiles;           // ceil(M / 128) * n_ntiles
    float eps;
    const float2* tab2;    // RoPE (c, s) per (t, i): the fp32 sums c_hi + c_lo, s_hi + s_lo
    const float2* gate;    // (B*T, Hkv) (g_hi, g_lo), value-embedding layers
    const __nv_bfloat16* ve;   // (B*T, Hkv, D), value-embedding layers
    __nv_bfloat16* qh;     // (B*T, H, D)
    __nv_bfloat16* kh;     // (B*T, Hkv, D)
    __nv_bfloat16* vp;     // (B*T, Hkv, D)
    int N;                 // (H + 2 Hkv) D output features
    int* sched_zero;       // two ints zeroed by block 0 (the attention kernel's counters), or null
    unsigned long long wait_limit_ns;
};

enum : unsigned int {
    kSiteQkvFull = 60, kSiteQkvEmpty = 61, kSiteQkvTFull = 62, kSiteQkvTEmpty = 63, kSiteQkvDrain = 64
};

// One head row of D fp32 accumulator values at tensor-memory address `taddr` (this warp's lanes):
// q / k heads get RoPE then RMS, v heads the gated value embedding; the result goes to `dst`
// (D bf16, 16-byte aligned).  Pair i of a q / k head is (i, i + D/2).  The tensor-memory loads
// are warp-collective, so every lane runs them; a lane whose token lies past the last one
// (`live` false) reads and writes no global memory.
template <int D, bool HAS_VE>
__device__ __forceinline__ void qkv_head_row(uint32_t taddr, bool is_v, bool live, int t, const QkvParams& p,
                                             const float2* g, const __nv_bfloat16* ve_row,
                                             __nv_bfloat16* dst) {
    constexpr int HALF = D / 2;
    if (!is_v) {
        // pass 1: sum of squares of the raw row (the rotation keeps it)
        float ss = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(taddr + (uint32_t)c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), ss);
        }
        const float r = (float)(1.0 / sqrt((double)ss / (double)D + (double)p.eps));
        // pass 2: rotate 16 pairs at a time, scale, round, store
        const float2* tab = p.tab2 + (long long)t * HALF;
#pragma unroll
        for (int i0 = 0; i0 < HALF; i0 += 16) {
            uint32_t a[16], b[16];
            __syncwarp();
            tmem_ld16(taddr + (uint32_t)i0, a);
            tmem_ld16(taddr + (uint32_t)(i0 + HALF), b);
            tmem_ld_wait();
            uint32_t wa[8], wb[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
                const float2 t0 = tab[i0 + e], t1 = tab[i0 + e + 1];
                const float c0 = t0.x, s0 = t0.y, c1 = t1.x, s1 = t1.y;
                const float a0 = __uint_as_float(a[e]), b0 = __uint_as_float(b[e]);
                const float a1 = __uint_as_float(a[e + 1]), b1 = __uint_as_float(b[e + 1]);
                wa[e >> 1] = pack_bf16x2((a0 * c0 - b0 * s0) * r, (a1 * c1 - b1 * s1) * r);
                wb[e >> 1] = pack_bf16x2((a0 * s0 + b0 * c0) * r, (a1 * s1 + b1 * c1) * r);
            }
            if (live) {
                uint4* da = reinterpret_cast<uint4*>(dst + i0);
                uint4* db = reinterpret_cast<uint4*>(dst + i0 + HALF);
                da[0] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
                da[1] = make_uint4(wa[4], wa[5], wa[6], wa[7]);
                db[0] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
                db[1] = make_uint4(wb[4], wb[5], wb[6], wb[7]);
            }
        }
    } else {
        float gv = 0.f;
        if constexpr (HAS_VE) {
            if (live) gv = g->x + g->y;
        }
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t v[16];
            __syncwarp();
            tmem_ld16(taddr + (uint32_t)c0, v);
            tmem_ld_wait();
            if (live) {
                float f[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) f[e] = __uint_as_float(v[e]);
                if constexpr (HAS_VE) {
                    const uint4* vr = reinterpret_cast<const uint4*>(ve_row + c0);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint4 u = vr[q];
                        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            f[8 * q + 2 * e] = fmaf(gv, __uint_as_float(w[e] << 16), f[8 * q + 2 * e]);
                            f[8 * q + 2 * e + 1] = fmaf(gv, __uint_as_float(w[e] & 0xffff0000u), f[8 * q + 2 * e + 1]);
                        }
                    }
                }
                uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
                d4[0] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                   pack_bf16x2(f[6], f[7]));
                d4[1] = make_uint4(pack_bf16x2(f[8], f[9]), pack_bf16x2(f[10], f[11]), pack_bf16x2(f[12], f[13]),
                                   pack_bf16x2(f[14], f[15]));
            }
        }
    }
}

template <int D, int BN, bool HAS_VE>
__global__ void __launch_bounds__(QkvCfg<BN>::THREADS, 1)
    qkv_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const QkvParams p) {
    using C = QkvCfg<BN>;
    constexpr int NS = C::NS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0u) {
        if (threadIdx.x == 0) record_error(kErrLayout, 0);
        return;
    }
    uint8_t* sRing = smem_raw;                     // NS x (x chunk | Wqkv chunk)
    uint64_t* bars = reinterpret_cast<uint64_t*>(sRing + NS * C::STAGE_BYTES);
    uint64_t* b_full = bars;                       // [NS]
    uint64_t* b_empty = bars + NS;                 // [NS]
    uint64_t* b_tfull = bars + 2 * NS;             // [2] accumulator complete
    uint64_t* b_tempty = bars + 2 * NS + 2;        // [2] accumulator read by the epilogue
    uint64_t* b_mdrain = bars + 2 * NS + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 5);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr uint32_t kEpiThreads = 32 * C::EPI_WARPS;
    if (threadIdx.x == 32) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(b_full + s), 1);
            mbar_init(smem_u32(b_empty + s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(b_tfull + i), 1);
            mbar_init(smem_u32(b_tempty + i), kEpiThreads);
        }
        mbar_init(smem_u32(b_mdrain), 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = p.wait_limit_ns;
    const int n_k = (p.C + C::BK - 1) / C::BK;
    if (blockIdx.x == 0 && threadIdx.x == 0 && p.sched_zero != nullptr) {
        p.sched_zero[0] = 0;
        p.sched_zero[1] = 0;
    }

    if (warp == 1) {
        // ============================== TMA producer ==============================
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t filled_phase[NS];
            bool filled[NS];
            for (int s = 0; s < NS; ++s) filled[s] = false, filled_phase[s] = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x) {
                const int m0 = (tile / p.n_ntiles) * C::BM;
                const int n0 = (tile % p.n_ntiles) * BN;
                for (int kc = 0; kc < n_k; ++kc) {
                    if (!(ok = mbar_wait(smem_u32(b_empty + stage), phase ^ 1u, lim, kSiteQkvEmpty))) break;
                    const uint32_t fb = smem_u32(b_full + stage);
                    uint8_t* st = sRing + stage * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(fb, (uint32_t)C::STAGE_BYTES);
                    tma_load_2d(smem_u32(st), &tm_x, fb, kc * C::BK, m0);
                    tma_load_2d(smem_u32(st + C::A_BYTES), &tm_w, fb, kc * C::BK, n0);
                    filled[stage] = true;
                    filled_phase[stage] = phase;
                    if (++stage == (uint32_t)NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < NS; ++s)
                if (filled[s]) mbar_wait(smem_u32(b_full + s), filled_phase[s], lim, kSiteQkvDrain);
        }
    } else if (warp == 0) {
        // ============================== MMA issuer ==============================
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false);   // A, B both K-major
            const uint64_t a0 = smem_desc_sw128(smem_u32(sRing), 16, 1024);
            const uint64_t b0 = smem_desc_sw128(smem_u32(sRing + C::A_BYTES), 16, 1024);
            uint32_t stage = 0, phase = 0, local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x, ++local) {
                const uint32_t buf = local & 1u;
                // the epilogue has read this buffer's previous tile (two tiles ago)
                if (local >= 2 && !(ok = mbar_wait(smem_u32(b_tempty + buf), ((local >> 1) - 1) & 1u, lim,
                                                  kSiteQkvTEmpty)))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + buf * (uint32_t)BN;
                for (int kc = 0; kc < n_k; ++kc) {
                    const uint32_t s = stage;
                    if (!(ok = mbar_wait(smem_u32(b_full + stage), phase, lim, kSiteQkvFull))) break;
                    if (++stage == (uint32_t)NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    const uint64_t so = (uint64_t)((s * C::STAGE_BYTES) >> 4);
#pragma unroll
                    for (int kk = 0; kk < C::BK / 16; ++kk)
                        mma_ss(d, a0 + so + (uint64_t)(kk * 2), b0 + so + (uint64_t)(kk * 2), idesc,
                               (kc > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(smem_u32(b_empty + s));
                }
                if (!ok) break;
                mma_commit(smem_u32(b_tfull + buf));
            }
            mma_commit(smem_u32(b_mdrain));
            mbar_wait(smem_u32(b_mdrain), 0, lim, kSiteQkvDrain);
        }
        __syncwarp();
    } else {
        // ================================ epilogue ================================
        const int blk = (warp - 2) >> 2;                 // 128-column block of the tile
        const int r = ((warp & 3) << 5) + lane;          // token row of the tile
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int HD = p.H * D, KD = p.Hkv * D;
        uint32_t local = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++local) {
            const uint32_t buf = local & 1u;
            const bool w = mbar_wait(smem_u32(b_tfull + buf), (local >> 1) & 1u, lim, kSiteQkvTFull);
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
            tc_fence_after();
            const int token = (tile / p.n_ntiles) * C::BM + r;
            const bool live = token < p.M;
            const long long tok = live ? token : 0;     // rows past the last token touch nothing
            const int t = (int)(tok % p.T);
            const int nb = (tile % p.n_ntiles) * BN + 128 * blk;   // first output feature of the block
            // the 128-column block holds 128 / D whole heads, all in one of q, k, v (warp-uniform)
            for (int hh = 0; hh < 128 / D; ++hh) {
                const int n = nb + hh * D;
                if (n >= p.N) break;                       // past the last head (warp-uniform)
                const uint32_t taddr = tmem + lane_base + buf * (uint32_t)BN + (uint32_t)(128 * blk + hh * D);
                if (n < HD) {
                    qkv_head_row<D, HAS_VE>(taddr, false, live, t, p, nullptr, nullptr, p.qh + tok * p.H * D + n);
                } else if (n < HD + KD) {
                    qkv_head_row<D, HAS_VE>(taddr, false, live, t, p, nullptr, nullptr,
                                            p.kh + tok * p.Hkv * D + (n - HD));
                } else {
                    const long long row = tok * p.Hkv + (n - HD - KD) / D;
                    qkv_head_row<D, HAS_VE>(taddr, true, live, t, p, HAS_VE ? p.gate + row : nullptr,
                                            HAS_VE ? p.ve + row * D : nullptr, p.vp + row * D);
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(b_tempty + buf));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace swa
