// attn_fwd.cuh -- causal sliding-window attention forward on the sm_100a tensor cores.
//
// What it computes ("Let's reproduce GPT-2 (124M)" notes, section 3 and section 19;
// intelliparadigm "GPT-2 for $73", section 3.2):
//   out[b,i,h,:] = sum_{j in J_i} softmax_j(qhat_i . khat_j / sqrt(D)) v'_j,
//   J_i = { j : 0 <= i - j < W },  lse[b,h,i] = ln sum_{j in J_i} exp(qhat_i . khat_j / sqrt(D)),
// on the RMS-normalised, rotated qhat/khat and the gated v' that the prologue wrote.
//
// Work item: one 128-row query tile of one (b, h).  The item walks the 128-row key/value tiles
// that intersect its window band [q0 - W + 1, q0 + 127]; tiles outside the band are never
// loaded.  The kernel is persistent: one CTA per SM takes items from a global counter (ordered in
// L2-sized chunks of (b, h) slices, heaviest first inside a chunk) until none is left.
// Warp roles (576 threads):
//   warp  0     TMEM allocator and the single thread that issues tcgen05.mma
//   warp  1     scheduler + TMA producer: the Q tile, then K_j, V_j through an NS-stage ring
//   warps 2-17  softmax + epilogue.  Warp w reaches the TMEM lanes 32 (w % 4) .. +31 (rows of the
//               tile) and takes key columns 32 c .. 32 c + 31 of them, c = (w - 2) / 4: four
//               threads share each row.
// Tensor memory: S(0) | S(1) (128 fp32 columns each) | O (D columns) | Q (D / 2 columns of bf16
// pairs).  Q is copied once per item from shared memory into tensor memory (tcgen05.cp), so the
// score products read only K from shared memory: with the TMA writes of K and V and the PV
// product's reads of V, shared-memory traffic is about the 128 bytes per clock the SM provides
// at the tensor rate.  The score products run one key tile ahead of the PV products:
// S_{j+1} = Q K_{j+1}^T goes into the buffer that held P_{j-1}, whose PV product was issued
// before it on the same in-order pipe, so the tensor pipe has a score product queued while the
// softmax of tile j is in progress.  P (bf16) of keys 32 c .. 32 c + 31 is written over S columns
// 32 c .. 32 c + 15, columns the same thread has just read, and fed to the PV product straight
// from tensor memory.
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
// Every exponential runs on MUFU (a polynomial on the FMA pipe is kept behind a zero mask: sending
// part of the pairs to it measured slower, the loop being bound by the issue of its products).
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
    static constexpr int NS = (D == 128) ? 4 : 11;     // K/V ring depth
    static constexpr int NSB = 2;                      // score buffers in tensor memory
    static constexpr int SMEM_Q = TILE_BYTES;
    static constexpr int SMEM_KV = NS * TILE_BYTES;
    static constexpr int SMEM_OUT = TILE_BYTES;        // output tile staged for the TMA store
    static constexpr int SMEM_BAR = 512;
    // Softmax threads per tile row (NQ) and the key columns each takes (CW).  Four is the most
    // that fits: 128 NQ softmax threads plus the MMA and producer warps must stay within 1024.
    static constexpr int NQ = 4;
    static constexpr int CW = 128 / NQ;
    static constexpr int SMEM_LX = NQ * 128 * 8;       // row-sum exchange between the NQ threads of a row
    // Dynamic shared memory is declared 1024-byte aligned (the 128-byte swizzle atom repeats every
    // 1024 bytes); the kernel checks the alignment on entry instead of reserving slack for it.
    static constexpr int SMEM_TOTAL = SMEM_Q + SMEM_KV + SMEM_OUT + SMEM_BAR + SMEM_LX;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_O = NSB * 128;
    static constexpr uint32_t COL_Q = COL_O + D;       // Q as bf16 pairs: D / 2 columns
    static constexpr int SOFTMAX_THREADS = 128 * NQ;
    static constexpr int SOFTMAX_WARPS = SOFTMAX_THREADS / 32;
    static constexpr int THREADS = 64 + SOFTMAX_THREADS;
    static_assert(CW == 16 || CW == 32, "softmax column split");
};

struct FwdParams {
    int B, T, H;
    int W;                 // effective window, 1..T
    int n_qtiles;          // ceil(T / 128)
    int n_items;           // n_qtiles * H * B
    int chunk_bh;          // (b, h) slices per scheduling chunk
    int G;                 // query heads per key/value head (1: multi-head; >1: grouped-query)
    float c1;              // log2(e) / sqrt(D): raw score -> log2 units
    float c2;              // M0 * log2(e)
    float m0;              // M0 (natural-log units), added back into the LSE
    __nv_bfloat16* out;    // (B,T,H,D)
    float* lse;            // (B,H,T) or null
    int* sched;            // [0] next item, [1] CTAs done; zero before the launch, reset after
    unsigned long long wait_limit_ns;
    const int* dstart;     // (B, T) start of each position's document (document mask), or null
};

// Wait sites recorded in the status word on timeout.
enum : unsigned int {
    kSiteQFull = 1, kSiteKvEmpty = 2, kSiteKvFull = 3, kSiteSFull = 4, kSitePFull = 5,
    kSiteOFull = 6, kSiteDrain = 7, kSiteQEmpty = 8, kSiteOEmpty = 9, kSiteItem = 10,
    kSiteRowSum = 11, kSiteOStage = 12
};

// Decoded work item: query tile [q0, q0 + 127] of (b, h) and the key tiles lo..hi of its band.
struct Item {
    int b, h, q0, lo, hi;
};

// Item order: chunks of `chunk_bh` (b, h) slices (their K/V fit in L2 together); inside a chunk,
// query tiles from the last (heaviest under the causal mask) to the first.
__device__ __forceinline__ Item decode_item(const FwdParams& p, int it) {
    Item m;
    const int per_chunk = p.chunk_bh * p.n_qtiles;
    const int chunk = it / per_chunk;
    const int rem = it - chunk * per_chunk;
    const int first_bh = chunk * p.chunk_bh;
    const int n_bh = min(p.chunk_bh, p.B * p.H - first_bh);
    const int qt = p.n_qtiles - 1 - rem / n_bh;
    const int bh = first_bh + rem % n_bh;
    m.b = bh / p.H;
    m.h = bh - m.b * p.H;
    m.q0 = qt * 128;
    m.lo = max(0, m.q0 - p.W + 1) / 128;
    m.hi = min(m.q0 + 127, p.T - 1) / 128;
    // Document mask: no key before the first query row's document start is visible to any row of
    // the tile (starts never decrease along the sequence), so those key tiles are skipped too.
    if (p.dstart != nullptr) m.lo = max(m.lo, p.dstart[(long long)m.b * p.T + m.q0] / 128);
    return m;
}

// One pair of raw scores -> P = 2^(s c1 - c2) on MUFU; accumulates the exact and the rounded
// sums (paired fp32) and returns the two P values as bf16 (toward zero) in one word, low half =
// first key.
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
// Pair j of every 8 consecutive key pairs takes the polynomial when bit j of this mask is set
// (unmasked tiles only); the rest go to MUFU.  All pairs go to MUFU: with the tile loop bound by
// the issue of its tensor-core products, sending 2 pairs of 8 to the polynomial measured 3-4%
// slower on B200 at D = 128 (the extra FMA-pipe instructions cost more than the MUFU time saved).
constexpr uint32_t kPolyPairMask = 0x00u;

struct PolyConsts {
    uint64_t shift, c3, c2, c1, c0;
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
        "sub.rn.f32x2 n, t, %7;\n\t"
        "sub.rn.f32x2 f, x, n;\n\t"
        "fma.rn.f32x2 q, %8, f, %9;\n\t"
        "fma.rn.f32x2 q, q, f, %10;\n\t"
        "fma.rn.f32x2 q, q, f, %11;\n\t"
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
        : "r"(s0), "r"(s1), "l"(c1x2), "l"(nc2x2), "l"(k.shift), "l"(k.c3), "l"(k.c2), "l"(k.c1),
          "l"(k.c0));
    return w;
}

template <int D, bool DOC = false>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0u) {   // uniform: every thread leaves before any barrier
        if (threadIdx.x == 0) record_error(kErrLayout, 0);
        return;
    }
    uint8_t* smem = smem_raw;
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + C::SMEM_Q;             // NS tiles
    uint8_t* sOut = sKV + C::SMEM_KV;            // output tile, same swizzled layout as the loads
    uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + C::SMEM_OUT);
    uint64_t* b_qfull = bars + 0;
    uint64_t* b_qempty = bars + 1;
    uint64_t* b_ofull = bars + 2;
    uint64_t* b_oempty = bars + 3;
    uint64_t* b_mdrain = bars + 4;               // MMA thread's final drain
    uint64_t* b_lxa = bars + 5;                  // columns 1-3 posted their row sums
    uint64_t* b_lxb = bars + 6;                  // column 0 posted the totals
    uint64_t* b_itfull = bars + 7;               // [2] scheduler slots
    uint64_t* b_itempty = bars + 9;              // [2]
    uint64_t* b_ostaged = bars + 11;             // every softmax thread wrote its part of the output tile
    uint64_t* b_ofree = bars + 12;               // the previous output tile has been read by its store
    uint64_t* b_sfull = bars + 13;               // [NSB]
    uint64_t* b_pfull = bars + 13 + C::NSB;      // [NSB]
    uint64_t* b_kvfull = bars + 13 + 2 * C::NSB;            // [NS]
    uint64_t* b_kvempty = bars + 13 + 2 * C::NSB + C::NS;   // [NS]
    int* s_item = reinterpret_cast<int*>(bars + 13 + 2 * C::NSB + 2 * C::NS);   // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_item + 2);
    float2* s_lx = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(bars) + C::SMEM_BAR);   // [4][128]
    static_assert(13 + 2 * C::NSB + 2 * C::NS <= (C::SMEM_BAR - 16) / 8, "barrier area");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // The MMA thread gets the lowest warp id: among ready warps the issue logic tends to favour
    // lower ids, and the tensor core idles whenever this thread waits for an issue slot.
    constexpr int kMmaWarp = 0;
    constexpr int kProducerWarp = 1;
    constexpr int kSoftmaxWarp0 = 2;
    constexpr uint32_t kItemConsumers = 1 + C::SOFTMAX_WARPS;  // the MMA thread and lane 0 of each softmax warp

    if (threadIdx.x == 32) {
        mbar_init(smem_u32(b_qfull), 1);
        mbar_init(smem_u32(b_qempty), 1);
        mbar_init(smem_u32(b_ofull), 1);
        mbar_init(smem_u32(b_oempty), C::SOFTMAX_THREADS);
        mbar_init(smem_u32(b_mdrain), 1);
        mbar_init(smem_u32(b_lxa), (C::NQ - 1) * 128);
        mbar_init(smem_u32(b_lxb), 128);
        mbar_init(smem_u32(b_ostaged), C::SOFTMAX_THREADS);
        mbar_init(smem_u32(b_ofree), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(b_itfull + i), 1);
            mbar_init(smem_u32(b_itempty + i), kItemConsumers);
        }
        for (int i = 0; i < C::NSB; ++i) {
            mbar_init(smem_u32(b_sfull + i), 1);
            mbar_init(smem_u32(b_pfull + i), C::SOFTMAX_THREADS);
        }
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
    // Launched as a programmatic dependent of the prologue: the setup above overlapped its tail;
    // nothing it wrote (qhat, khat, v', the item counter) is touched before this wait.
    grid_dependency_wait();

    if (warp == kProducerWarp) {
        // ========================= scheduler + TMA producer =========================
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t filled_phase[C::NS];
            bool filled[C::NS];
            for (int s = 0; s < C::NS; ++s) filled[s] = false, filled_phase[s] = 0;
            uint32_t q_uses = 0;
            bool ok = true;
            auto load_kv = [&](const CUtensorMap* tm, const Item& m, int j) -> bool {
                if (!mbar_wait(smem_u32(b_kvempty + stage), phase ^ 1u, lim, kSiteKvEmpty)) return false;
                const uint32_t fb = smem_u32(b_kvfull + stage);
                mbar_arrive_expect_tx(fb, (uint32_t)C::TILE_BYTES);
                for (int ch = 0; ch < C::NCHUNK; ++ch)
                    tma_load_4d(smem_u32(sKV + stage * C::TILE_BYTES + ch * C::CHUNK_BYTES), tm, fb, ch * 64,
                                m.h / p.G, j * C::BN, m.b);
                filled[stage] = true;
                filled_phase[stage] = phase;
                if (++stage == (uint32_t)C::NS) {
                    stage = 0;
                    phase ^= 1u;
                }
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
                // Warm L2 with this item's query tile while the previous item finishes.
                for (int ch = 0; ch < C::NCHUNK; ++ch) tma_prefetch_4d(&tm_q, ch * 64, m.h, m.q0, m.b);
                if (q_uses > 0 && !(ok = mbar_wait(smem_u32(b_qempty), (q_uses - 1) & 1u, lim, kSiteQEmpty)))
                    break;
                {
                    const uint32_t qb = smem_u32(b_qfull);
                    mbar_arrive_expect_tx(qb, (uint32_t)C::TILE_BYTES);
                    for (int ch = 0; ch < C::NCHUNK; ++ch)
                        tma_load_4d(smem_u32(sQ + ch * C::CHUNK_BYTES), &tm_q, qb, ch * 64, m.h, m.q0, m.b);
                    ++q_uses;
                }
                // The MMA thread's order: K_lo, then K_{j+1}, V_j for each key tile j.
                ok = load_kv(&tm_k, m, m.lo);
                for (int j = m.lo; ok && j <= m.hi; ++j)
                    ok = (j + 1 > m.hi || load_kv(&tm_k, m, j + 1)) && load_kv(&tm_v, m, j);
            }
            // The last CTA to run out of items resets the counters for the next launch.
            if (ok && atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
                p.sched[0] = 0;
                p.sched[1] = 0;
            }
            // Drain: every copy this thread started has landed before the CTA may exit.
            if (q_uses > 0) mbar_wait(smem_u32(b_qfull), (q_uses - 1) & 1u, lim, kSiteDrain);
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
            const uint32_t d_o = tmem + C::COL_O;
            uint32_t stage = 0, phase = 0;
            uint32_t s_cnt = 0, s_buf = 0;   // score products issued; buffer of the next one
            uint32_t p_cnt = 0, p_buf = 0;   // PV products issued; buffer they read
            uint32_t uses = 0;               // items done
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
            // S = Q K_j^T : M=128, N=BN, K=D in steps of 16; Q (A) from tensor memory, 8 columns per
            // step; K (B) from shared memory, 32 bytes inside a 128-byte swizzle chunk per step (the
            // descriptor start address advances in 16-byte units).  Then release the K slot.
            auto s_step = [&](int j) -> bool {
                (void)j;
                uint32_t sk = 0;
                if (!acquire(sk)) return false;
                const uint64_t db = dkv + (uint64_t)((sk * C::TILE_BYTES) >> 4);
                const uint32_t d = tmem + s_buf * 128u;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4;
                    mma_ts(d, tmem + C::COL_Q + 8u * kk, db + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(b_sfull + s_buf));
                mma_commit(smem_u32(b_kvempty + sk));
                ++s_cnt;
                if (++s_buf == (uint32_t)C::NSB) s_buf = 0;
                return true;
            };
            // O += P_j V_j : M=128, N=D, K=BN in steps of 16 key rows.  P from tensor memory (keys
            // 32 c + i at column 32 c + i / 2 of its score buffer), V MN-major from shared memory.
            // The item's first PV waits until the previous epilogue has read O.
            auto pv_step = [&](const Item& m, int j) -> bool {
                uint32_t sv = 0;
                if (!acquire(sv)) return false;
                if (!mbar_wait(smem_u32(b_pfull + p_buf), (p_cnt / C::NSB) & 1u, lim, kSitePFull)) return false;
                if (j == m.lo && uses > 0 && !mbar_wait(smem_u32(b_oempty), (uses - 1) & 1u, lim, kSiteOEmpty))
                    return false;
                tc_fence_after();
                const uint32_t pa = tmem + p_buf * 128u;
                const uint64_t db = dv + (uint64_t)((sv * C::TILE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ts(d_o, pa + (uint32_t)(C::CW * (16 * kk / C::CW) + (16 * kk % C::CW) / 2),
                           db + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv, (j > m.lo || kk > 0) ? 1u : 0u);
                mma_commit(smem_u32(b_kvempty + sv));
                if (j == m.hi) mma_commit(smem_u32(b_ofull));
                ++p_cnt;
                if (++p_buf == (uint32_t)C::NSB) p_buf = 0;
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
                // Q into tensor memory (after the previous item's score products on the same pipe),
                // then its shared-memory buffer goes back to the producer.
                if (!(ok = mbar_wait(smem_u32(b_qfull), uses & 1u, lim, kSiteQFull))) break;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tmem_cp_128x256b(tmem + C::COL_Q + 8u * kk,
                                     dq + (uint64_t)(((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4));
                mma_commit(smem_u32(b_qempty));
                ok = s_step(m.lo);
                for (int j = m.lo; ok && j <= m.hi; ++j)
                    ok = (j + 1 > m.hi || s_step(j + 1)) && pv_step(m, j);
                ++uses;
            }
            // Drain: every tensor-core operation issued above has finished before teardown.
            mma_commit(smem_u32(b_mdrain));
            mbar_wait(smem_u32(b_mdrain), 0, lim, kSiteDrain);
        }
        __syncwarp();
    } else {
        // ============================ softmax + epilogue ============================
        const int cq = (warp - kSoftmaxWarp0) >> 2;   // key / output column quarter
        // A warp reaches the TMEM lanes of its quarter, 32 (warp % 4) .. + 31: row r of the tile.
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
        uint32_t s_cnt = 0, s_buf = 0, o_uses = 0;
        // one thread issues the output tile's TMA store
        const bool is_store = (warp == kSoftmaxWarp0 && lane == 0);
        bool ok = true;

        // The k-th item from the scheduler's slots (k & 1); -1 when none is left.
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
            const int qi = m.q0 + r;              // this thread's query position
            // Document mask: this row's document start, and the largest start among the warp's
            // rows (warp-uniform test of whether a key block needs the per-element mask).
            int ds = 0, ds_w = 0;
            if constexpr (DOC) {
                ds = __ldg(p.dstart + (long long)m.b * p.T + min(qi, p.T - 1));
                ds_w = __reduce_max_sync(0xffffffffu, ds);
            }
            uint64_t l2[4], lr2[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) l2[a] = lr2[a] = 0ull;
            for (int j = m.lo; j <= m.hi; ++j) {
                const uint32_t buf = s_buf;
                const bool w = mbar_wait(smem_u32(b_sfull + buf), (s_cnt / C::NSB) & 1u, lim, kSiteSFull);
                ok = __all_sync(0xffffffffu, w);
                if (!ok) break;
                ++s_cnt;
                if (++s_buf == (uint32_t)C::NSB) s_buf = 0;
                tc_fence_after();
                const int k0 = j * C::BN + C::CW * cq;   // first key of this thread's CW columns
                const bool need_mask =
                    (k0 + C::CW - 1 > m.q0) || (m.q0 + C::BM - 1 - k0 >= p.W) || (DOC && k0 < ds_w);
                const uint32_t colS = buf * 128u + (uint32_t)(C::CW * cq);
                // The 32 scores in two 16-column blocks, both loaded before any arithmetic; P of
                // the 32 keys packs into 16 words written over the first 16 of these columns.
                uint32_t sq[C::CW / 16][16];
                uint32_t pk[C::CW / 2];
                auto block = [&](const uint32_t (&sv)[16], int cbase, int pkbase) {
                    if (!need_mask) {
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const int a = (e >> 1) & 3;
                            pk[pkbase + (e >> 1)] =
                                ((kPolyPairMask >> (e >> 1)) & 1u)
                                    ? softmax_pair_poly(sv[e], sv[e + 1], c1x2, nc2x2, pc, l2[a], lr2[a])
                                    : softmax_pair_mufu(sv[e], sv[e + 1], c1x2, nc2x2, l2[a], lr2[a]);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const int kv = k0 + cbase + e;
                            // masked scores become -inf in log2 units, so exp gives exactly 0
                            const uint32_t m0 = ((unsigned)(qi - kv) >= (unsigned)p.W || (DOC && kv < ds))
                                                    ? 0xff800000u : sv[e];
                            const uint32_t m1 = ((unsigned)(qi - kv - 1) >= (unsigned)p.W || (DOC && kv + 1 < ds))
                                                    ? 0xff800000u : sv[e + 1];
                            pk[pkbase + (e >> 1)] =
                                softmax_pair_mufu(m0, m1, c1x2, nc2x2, l2[e >> 1 & 3], lr2[e >> 1 & 3]);
                        }
                    }
                };
                tmem_ld16(tmem + lane_base + colS + 0, sq[0]);
                if constexpr (C::CW == 32) tmem_ld16(tmem + lane_base + colS + 16, sq[C::CW / 16 - 1]);
                tmem_ld_wait();
                block(sq[0], 0, 0);
                if constexpr (C::CW == 32) {
                    block(sq[C::CW / 16 - 1], 16, 8);
                    tmem_st16(tmem + lane_base + colS + 0, *reinterpret_cast<const uint32_t(*)[16]>(pk));
                } else {
                    tmem_st8(tmem + lane_base + colS + 0, *reinterpret_cast<const uint32_t(*)[8]>(pk));
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(smem_u32(b_pfull + buf));
            }
            if (!ok) break;
            // This thread's partial row sums (few registers stay live across the next step).
            float l = 0.f, lr = 0.f;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                float u0, u1, w0, w1;
                f2_unpack(l2[a], u0, u1);
                f2_unpack(lr2[a], w0, w1);
                l += u0 + u1;
                lr += w0 + w1;
            }
            // The next item (read early: its slot frees the scheduler's next publication).
            ++k;
            const int it_next = fetch(k);
            if (!ok) break;
            {
                const bool w = mbar_wait(smem_u32(b_ofull), o_uses & 1u, lim, kSiteOFull);
                ok = __all_sync(0xffffffffu, w);
            }
            if (!ok) break;
            tc_fence_after();
            // Read this thread's quarter of the O row, then release O to the next item.
            constexpr int OQ = D / C::NQ;         // output columns per thread: 8 to 32
            uint32_t ov[OQ];
            if constexpr (OQ == 32) {
                tmem_ld16(tmem + lane_base + C::COL_O + (uint32_t)(OQ * cq), *reinterpret_cast<uint32_t(*)[16]>(ov));
                tmem_ld16(tmem + lane_base + C::COL_O + (uint32_t)(OQ * cq) + 16u,
                          *reinterpret_cast<uint32_t(*)[16]>(ov + 16));
            } else if constexpr (OQ == 16) {
                tmem_ld16(tmem + lane_base + C::COL_O + (uint32_t)(OQ * cq), *reinterpret_cast<uint32_t(*)[16]>(ov));
            } else {
                tmem_ld8(tmem + lane_base + C::COL_O + (uint32_t)(OQ * cq), *reinterpret_cast<uint32_t(*)[8]>(ov));
            }
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(smem_u32(b_oempty));
            ++o_uses;
            // Row sums: columns 1-3 post their partial sums, column 0 adds them and posts the
            // totals; two mbarriers with bounded waits order the exchange.
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
                for (int c = 1; c < C::NQ; ++c) {
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
            // The output tile goes through shared memory (the 128-byte-swizzled layout of the
            // tensor map) and leaves in one TMA store, which also drops rows past T.  Before the
            // tile is rewritten, the store thread confirms that the previous store has read it.
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
                const int col0 = OQ * cq;                        // first output feature of this thread
                uint8_t* rowp = sOut + (col0 >> 6) * C::CHUNK_BYTES + r * 128;
                const int u0 = (col0 & 63) >> 3;                 // first 16-byte unit in the 128-byte row
#pragma unroll
                for (int e = 0; e < OQ / 8; ++e)
                    *reinterpret_cast<uint4*>(rowp + (((u0 + e) ^ (r & 7)) << 4)) =
                        make_uint4(w16[4 * e], w16[4 * e + 1], w16[4 * e + 2], w16[4 * e + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(b_ostaged));
            if (is_store) {
                if (mbar_wait(smem_u32(b_ostaged), e_idx & 1u, lim, kSiteOStage)) {
                    for (int ch = 0; ch < C::NCHUNK; ++ch)
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

    // The output stores have completed before the CTA exits.
    if (warp == kSoftmaxWarp0 && lane == 0) bulk_wait_all();
    // ---- teardown: all tensor-memory traffic of this CTA is finished before the free.
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace swa
