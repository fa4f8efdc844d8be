// swa_attn.cu -- host side of the C ABI declared in include/swa_attn.h: argument checks,
// workspace management, TMA descriptors and the two kernel launches (prologue, attention).
// All kernels are in this translation unit (ptx.cuh, prologue.cuh, attn_fwd.cuh, attn_bwd.cuh,
// decode.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "swa_attn.h"
#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "decode.cuh"
#include "prologue.cuh"
#include "qkv_gemm.cuh"
#include "docmask.cuh"

// ------------------------------------------------------------------ failure-detection self-test

namespace swa {
// Waits, through the same bounded wait the kernels use, on an mbarrier that nothing ever
// completes: after `limit_ns` the wait gives up and records a timeout at site kSiteSelfTest.
constexpr unsigned int kSiteSelfTest = 30;
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    mbar_wait(smem_u32(&bar), 0u, limit_ns, kSiteSelfTest);
}
}  // namespace swa

namespace {

constexpr int kVersion = 100;   // 0.1.0

// ------------------------------------------------------------------ configuration knobs

std::mutex g_cache_mu;                          // guards the per-device workspace cache
std::atomic<unsigned long long> g_wait_limit_ns{0};   // 0 = not yet initialised

unsigned long long wait_limit_ns() {
    unsigned long long v = g_wait_limit_ns.load(std::memory_order_relaxed);
    if (v != 0) return v;
    long ms = 2000;
    if (const char* e = std::getenv("SWA_WAIT_LIMIT_MS")) {
        const long x = std::strtol(e, nullptr, 10);
        if (x >= 1) ms = x;
    }
    unsigned long long expected = 0;
    const unsigned long long want = (unsigned long long)ms * 1000000ull;
    g_wait_limit_ns.compare_exchange_strong(expected, want);
    return g_wait_limit_ns.load(std::memory_order_relaxed);
}

// ---------------------------------------------------------------------- argument checks

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Shape {
    int B, T, H, D;
    long long n;          // B*T*H*D
    int Hkv;              // key/value heads (H unless grouped-query attention)
};

int check_sizes(int B, int T, int H, int D, Shape* s) {
    if (B < 1 || T < 1 || H < 1) return SWA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
    const long long n = (long long)B * T * H * D;
    if (n >= (1ll << 31)) return SWA_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return SWA_ERR_UNSUPPORTED;   // grid y/z limits
    *s = Shape{B, T, H, D, n, H};
    return SWA_OK;
}

// Grouped-query attention: Hkv key/value heads, 1 <= Hkv <= H, Hkv divides H.
int check_kv_heads(int Hkv, Shape* s) {
    if (Hkv < 1 || Hkv > s->H || (s->H % Hkv) != 0) return SWA_ERR_INVALID_ARG;
    s->Hkv = Hkv;
    return SWA_OK;
}

int check_layer_args(const void* q, const void* k, const void* v, const void* ve,
                     const void* gate_x, const void* Wg, float rope_base, float eps) {
    if (!q || !k || !v) return SWA_ERR_INVALID_ARG;
    const int n_ve = (ve != nullptr) + (gate_x != nullptr) + (Wg != nullptr);
    if (n_ve != 0 && n_ve != 3) return SWA_ERR_INVALID_ARG;
    if (!std::isfinite(rope_base) || !(rope_base > 0.f)) return SWA_ERR_INVALID_ARG;
    if (!std::isfinite(eps) || eps < 0.f) return SWA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return SWA_ERR_MISALIGNED;
    if (n_ve == 3 && (!aligned(ve, 16) || !aligned(gate_x, 2) || !aligned(Wg, 2)))
        return SWA_ERR_MISALIGNED;
    return SWA_OK;
}

int check_outputs(const void* out, const float* lse) {
    if (!out) return SWA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || (lse && !aligned(lse, 4))) return SWA_ERR_MISALIGNED;
    return SWA_OK;
}

// ---------------------------------------------------------------------- workspace layout

constexpr size_t kAlign = 1024;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct WsLayout {
    size_t qh, kh, vp, gate, tab32, tab64, sched, dstart, total;
};

// Grid of one prologue pass over `rows` rows: 256-thread blocks, D / 8 threads per row, at most
// one wave of three resident blocks per SM (each block repairs its own list at its end).
long long prologue_blocks(long long rows, int D) {
    return std::max<long long>(1, std::min<long long>((rows * (D / 8) + 255) / 256, 148ll * 3));
}

// qhat | khat | v' and gate (value-embedding layers only) | RoPE table fp32 pieces |
// RoPE table fp64 | attention scheduler counters | document starts (B, T) int32
// (document-masked calls only), each section 1024-byte aligned.
WsLayout ws_layout(const Shape& s, bool has_ve, bool has_doc = false) {
    WsLayout w{};
    const size_t tensor = round_up((size_t)s.n * 2);
    const size_t kv_tensor = round_up((size_t)s.B * s.T * s.Hkv * s.D * 2);
    const size_t pairs = (size_t)s.T * (s.D / 2);
    w.qh = 0;
    w.kh = w.qh + tensor;
    w.vp = w.kh + kv_tensor;
    w.gate = w.vp + (has_ve ? kv_tensor : 0);
    w.tab32 = w.gate + (has_ve ? round_up((size_t)s.B * s.T * s.Hkv * sizeof(float2)) : 0);
    w.tab64 = w.tab32 + round_up(pairs * sizeof(float4));
    w.sched = w.tab64 + round_up(pairs * sizeof(double2));
    w.dstart = w.sched + kAlign;
    w.total = w.dstart + (has_doc ? round_up((size_t)s.B * s.T * sizeof(int)) : 0);
    return w;
}

// ---------------------------------------------------------------------------- device

int g_num_sms[64] = {0};

// Dynamic shared memory of every instantiation of the fused projection kernel (set on the first
// fused-projection call on each device, so the other entry points never depend on it).
bool set_qkv_smem() {
    const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    return cudaFuncSetAttribute(swa::qkv_gemm_kernel<128, 256, true>, a, swa::QkvCfg<256>::SMEM_TOTAL) == cudaSuccess &&
           cudaFuncSetAttribute(swa::qkv_gemm_kernel<128, 256, false>, a, swa::QkvCfg<256>::SMEM_TOTAL) == cudaSuccess &&
           cudaFuncSetAttribute(swa::qkv_gemm_kernel<128, 128, true>, a, swa::QkvCfg<128>::SMEM_TOTAL) == cudaSuccess &&
           cudaFuncSetAttribute(swa::qkv_gemm_kernel<128, 128, false>, a, swa::QkvCfg<128>::SMEM_TOTAL) == cudaSuccess &&
           cudaFuncSetAttribute(swa::qkv_gemm_kernel<64, 256, true>, a, swa::QkvCfg<256>::SMEM_TOTAL) == cudaSuccess &&
           cudaFuncSetAttribute(swa::qkv_gemm_kernel<64, 256, false>, a, swa::QkvCfg<256>::SMEM_TOTAL) == cudaSuccess &&
           cudaFuncSetAttribute(swa::qkv_gemm_kernel<64, 128, true>, a, swa::QkvCfg<128>::SMEM_TOTAL) == cudaSuccess &&
           cudaFuncSetAttribute(swa::qkv_gemm_kernel<64, 128, false>, a, swa::QkvCfg<128>::SMEM_TOTAL) == cudaSuccess;
}

// Device `dev` must be compute capability 10.0; its SM count goes to g_num_sms[dev].  On such a
// device, raises the dynamic shared memory limit of every kernel that uses more than 48 KB.
// Returns 1 (ready), 2 (not sm_100) or a negative status.
int check_device(int dev) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return SWA_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return 2;
    const int smem_attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
    if (cudaFuncSetAttribute(swa::attn_fwd_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             swa::FwdCfg<64>::SMEM_TOTAL) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_fwd_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             swa::FwdCfg<128>::SMEM_TOTAL) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_fwd_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             swa::FwdCfg<64>::SMEM_TOTAL) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_fwd_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             swa::FwdCfg<128>::SMEM_TOTAL) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_bwd_dq_kernel<64>, (cudaFuncAttribute)smem_attr,
                             swa::BwdCfg<64>::DQ_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_bwd_dq_kernel<128>, (cudaFuncAttribute)smem_attr,
                             swa::BwdCfg<128>::DQ_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_bwd_dkv_kernel<64>, (cudaFuncAttribute)smem_attr,
                             swa::BwdCfg<64>::KV_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_bwd_dkv_kernel<128>, (cudaFuncAttribute)smem_attr,
                             swa::BwdCfg<128>::KV_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_bwd_dq_kernel<64, true>, (cudaFuncAttribute)smem_attr,
                             swa::BwdCfg<64>::DQ_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_bwd_dq_kernel<128, true>, (cudaFuncAttribute)smem_attr,
                             swa::BwdCfg<128>::DQ_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_bwd_dkv_kernel<64, true>, (cudaFuncAttribute)smem_attr,
                             swa::BwdCfg<64>::KV_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::attn_bwd_dkv_kernel<128, true>, (cudaFuncAttribute)smem_attr,
                             swa::BwdCfg<128>::KV_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::decode_attn_kernel<64>, (cudaFuncAttribute)smem_attr,
                             swa::DecCfg<64>::SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(swa::decode_attn_kernel<128>, (cudaFuncAttribute)smem_attr,
                             swa::DecCfg<128>::SMEM) != cudaSuccess) {
        cudaGetLastError();
        return SWA_ERR_CUDA;
    }
    return 1;
}

// Per-device state of device_ready: 0 not yet checked, 1 ready, 2 unsupported.  The first call
// on a device checks it under g_dev_mu; g_num_sms[dev] is written before the state is published.
std::mutex g_dev_mu;
std::atomic<int> g_dev_state[64];

int device_ready(int* dev_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SWA_ERR_NO_DEVICE;
    }
    if (dev < 0 || dev >= 64) return SWA_ERR_UNSUPPORTED;
    int state = g_dev_state[dev].load(std::memory_order_acquire);
    if (state == 0) {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        state = g_dev_state[dev].load(std::memory_order_relaxed);
        if (state == 0 && (state = check_device(dev)) < 0) return state;
        g_dev_state[dev].store(state, std::memory_order_release);
    }
    *dev_out = dev;
    return state == 1 ? SWA_OK : SWA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------- TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// A (B,T,heads,D) bf16 tensor seen as 4-D {D, heads, T, B}; box = 64 features x 1 head x 128 positions,
// 128-byte swizzle (the canonical K-major / MN-major shared-memory atom of the tensor core).
// Positions past T read as zeros.
bool make_tile_map(CUtensorMap* m, const void* base, const Shape& s, int heads) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)s.D, (cuuint64_t)heads, (cuuint64_t)s.T, (cuuint64_t)s.B};
    const cuuint64_t strides[3] = {(cuuint64_t)s.D * 2, (cuuint64_t)heads * s.D * 2,
                                   (cuuint64_t)s.T * heads * s.D * 2};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------- launches

swa::FastDiv make_fastdiv(int d) {
    int l = 0;
    while ((1ll << l) < d) ++l;          // ceil(log2 d)
    const int k = 32 + l;
    swa::FastDiv f;
    f.m = (unsigned long long)((((unsigned __int128)1 << k) + (unsigned)d - 1) / (unsigned)d);
    f.k = k;
    f.d = d;
    return f;
}

// A launch that may start while the kernel before it on the stream still runs (programmatic
// dependent launch): the kernel waits (griddepcontrol.wait) before it touches memory that kernel
// wrote, so only the launch latency and its own setup overlap.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, args...);
}

// fused: the fused projection's table, (c, s) as fp32 sums in the section that otherwise holds the
// fp64 table (which only the prologue's repairs read).
int launch_rope_table(uint8_t* ws, const WsLayout& L, const Shape& s, float rope_base, cudaStream_t st,
                      bool fused = false) {
    const long long n = (long long)s.T * (s.D / 2);
    const int threads = 256;
    const long long blocks = std::min<long long>((n + threads - 1) / threads, 148ll * 16);
    swa::rope_table_kernel<<<(unsigned)blocks, threads, 0, st>>>(
        reinterpret_cast<float4*>(ws + L.tab32), fused ? nullptr : reinterpret_cast<double2*>(ws + L.tab64),
        fused ? reinterpret_cast<float2*>(ws + L.tab64) : nullptr, s.T, s.D, (double)rope_base);
    return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int launch_prologue(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                    const void* Wg, uint8_t* ws, const WsLayout& L, const Shape& s, float eps,
                    cudaStream_t st) {
    using bf = __nv_bfloat16;
    const bool has_ve = ve != nullptr;
    const int n_rows = s.B * s.T * s.H;
    const int n_kv_rows = s.B * s.T * s.Hkv;
    const swa::FastDiv divH = make_fastdiv(s.H), divT = make_fastdiv(s.T);
    float2* gate = reinterpret_cast<float2*>(ws + L.gate);
    const int threads = 256;
    const long long blocks = prologue_blocks(n_rows, s.D);
    if (has_ve) {
        const int n_tok = s.B * s.T;
        const int gblocks = (int)std::min<long long>(((long long)n_tok + 127) / 128, 148ll * 16);
        const int wg_smem = 32 * s.Hkv * (int)sizeof(double) <= 48 * 1024;
        swa::gate_kernel<<<gblocks, 128, wg_smem ? 32 * s.Hkv * sizeof(double) : 0, st>>>(
            static_cast<const bf*>(gate_x), static_cast<const bf*>(Wg), gate, n_tok, s.Hkv, 32, wg_smem);
    }
    const bf* qp = static_cast<const bf*>(q);
    const bf* kp = static_cast<const bf*>(k);
    const bf* vpi = static_cast<const bf*>(v);
    const bf* vep = static_cast<const bf*>(ve);
    bf* qh = reinterpret_cast<bf*>(ws + L.qh);
    bf* kh = reinterpret_cast<bf*>(ws + L.kh);
    bf* vp = reinterpret_cast<bf*>(ws + L.vp);
    const float4* t32 = reinterpret_cast<const float4*>(ws + L.tab32);
    const double2* t64 = reinterpret_cast<const double2*>(ws + L.tab64);
    int* sched = reinterpret_cast<int*>(ws + L.sched);
    const unsigned g = (unsigned)blocks;
    const double e = (double)eps;
    if (s.Hkv != s.H) {
        // Grouped-query attention: the query rows (H heads) and the key/value rows (Hkv heads) are
        // two passes over their own rows.
        const swa::FastDiv divK = make_fastdiv(s.Hkv);
        const unsigned gk = (unsigned)prologue_blocks(n_kv_rows, s.D);
#define SWA_PRO_GQA(DD, VE)                                                                                  \
    swa::prologue_kernel<DD, VE, 1><<<g, threads, 0, st>>>(qp, kp, vpi, vep, gate, qh, kh, vp, t32, t64, sched, \
                                                           n_rows, s.T, s.H, divT, divH, e);                 \
    swa::prologue_kernel<DD, VE, 2><<<gk, threads, 0, st>>>(qp, kp, vpi, vep, gate, qh, kh, vp, t32, t64, sched, \
                                                            n_kv_rows, s.T, s.Hkv, divT, divK, e)
        if (s.D == 128) {
            if (has_ve) {
                SWA_PRO_GQA(128, true);
            } else {
                SWA_PRO_GQA(128, false);
            }
        } else {
            if (has_ve) {
                SWA_PRO_GQA(64, true);
            } else {
                SWA_PRO_GQA(64, false);
            }
        }
#undef SWA_PRO_GQA
        return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
    }
#define SWA_PRO(DD, VE)                                                                                          \
    launch_pdl(swa::prologue_kernel<DD, VE, 3>, dim3(g), dim3(threads), 0, st, qp, kp, vpi, vep, (const float2*)gate, \
               qh, kh, vp, t32, t64, sched, n_rows, s.T, s.H, divT, divH, e)
    if (s.D == 128) {
        if (has_ve) SWA_PRO(128, true); else SWA_PRO(128, false);
    } else {
        if (has_ve) SWA_PRO(64, true); else SWA_PRO(64, false);
    }
#undef SWA_PRO
    return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

// The attention kernel on the workspace's qhat, khat (and v' on value-embedding layers; `v` itself
// otherwise).  dstart: the document starts (B, T) of a document-masked call, or null.
int launch_attention(int dev, const void* v, bool has_ve, void* out, float* lse, const Shape& s, int window,
                     uint8_t* ws, const WsLayout& L, cudaStream_t st, const int* dstart = nullptr) {
    CUtensorMap tq, tk, tv, to;
    const void* vsrc = has_ve ? static_cast<const void*>(ws + L.vp) : v;
    const void* qsrc = ws + L.qh;
    // q and out have H heads, k and v Hkv heads
    if (!make_tile_map(&tq, qsrc, s, s.H) || !make_tile_map(&tk, ws + L.kh, s, s.Hkv) ||
        !make_tile_map(&tv, vsrc, s, s.Hkv) || !make_tile_map(&to, out, s, s.H))
        return SWA_ERR_CUDA;
    swa::FwdParams p{};
    p.B = s.B;
    p.T = s.T;
    p.H = s.H;
    p.W = (window <= 0 || window >= s.T) ? s.T : window;
    p.G = s.H / s.Hkv;
    p.n_qtiles = (s.T + 127) / 128;
    p.n_items = p.n_qtiles * s.H * s.B;
    // Scheduling chunks of (b, h) slices whose K/V (about 4 T D bytes each) fit in ~40 MB of L2.
    const long long slice_bytes = 4ll * s.T * s.D;
    p.chunk_bh = (int)std::max<long long>(1, std::min<long long>((40ll << 20) / slice_bytes, (long long)s.B * s.H));
    const double log2e = 1.4426950408889634;
    const double m0 = std::sqrt((double)s.D) * (1.0 + 1.0 / 64.0);
    p.c1 = (float)(log2e / std::sqrt((double)s.D));
    p.c2 = (float)(m0 * log2e);
    p.m0 = (float)m0;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.sched = reinterpret_cast<int*>(ws + L.sched);
    p.wait_limit_ns = wait_limit_ns();
    p.dstart = dstart;
    const dim3 grid((unsigned)std::min(p.n_items, g_num_sms[dev]));
#define SWA_ATTN(DD, DC) \
    launch_pdl(swa::attn_fwd_kernel<DD, DC>, grid, dim3(swa::FwdCfg<DD>::THREADS), swa::FwdCfg<DD>::SMEM_TOTAL, st, tq, tk, \
               tv, to, p)
    if (s.D == 128) {
        if (dstart) SWA_ATTN(128, true); else SWA_ATTN(128, false);
    } else {
        if (dstart) SWA_ATTN(64, true); else SWA_ATTN(64, false);
    }
#undef SWA_ATTN
    return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

// --------------------------------------------------------------- fused q/k/v projection

// A (rows, cols) row-major bf16 matrix as a 2-D tensor map {cols, rows}; box = 64 columns (one
// 128-byte swizzle atom) x box_rows rows.  Rows and columns past the end read as zeros.
bool make_matrix_map(CUtensorMap* m, const void* base, long long rows, int cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int check_qkv_args(const void* x, const void* Wqkv, const void* ve, const void* Wg, const Shape& s, int C,
                   float rope_base, float eps) {
    if (!x || !Wqkv) return SWA_ERR_INVALID_ARG;
    if ((ve == nullptr) != (Wg == nullptr)) return SWA_ERR_INVALID_ARG;
    if (C < 8 || (C % 8) != 0) return SWA_ERR_UNSUPPORTED;   // 16-byte rows for the tensor maps
    if ((long long)s.B * s.T * C >= (1ll << 31)) return SWA_ERR_UNSUPPORTED;   // int32 indexing of x
    if (ve != nullptr && C < 32) return SWA_ERR_INVALID_ARG;  // the gate reads 32 channels
    if (!std::isfinite(rope_base) || !(rope_base > 0.f)) return SWA_ERR_INVALID_ARG;
    if (!std::isfinite(eps) || eps < 0.f) return SWA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(Wqkv, 16) || (ve && (!aligned(ve, 16) || !aligned(Wg, 2))))
        return SWA_ERR_MISALIGNED;
    return SWA_OK;
}

// Gate (value-embedding layers), then the fused projection kernel writing qhat, khat, v' to
// qh / kh / vp.  The RoPE table must already be in the workspace.
int launch_qkv(int dev, const void* x, const void* Wqkv, const void* ve, const void* Wg, int C, const Shape& s,
               float eps, uint8_t* ws, const WsLayout& L, void* qh, void* kh, void* vp, int* sched_zero,
               cudaStream_t st) {
    using bf = __nv_bfloat16;
    const bool has_ve = ve != nullptr;
    const long long M = (long long)s.B * s.T;
    if (M * C >= (1ll << 31) || M >= (1ll << 31) / std::max(1, s.H * s.D)) return SWA_ERR_UNSUPPORTED;
    {
        static std::once_flag once[64];
        static bool ok[64] = {false};
        std::call_once(once[dev], [&] { ok[dev] = set_qkv_smem(); });
        if (!ok[dev]) {
            cudaGetLastError();
            return SWA_ERR_CUDA;
        }
    }
    float2* gate = reinterpret_cast<float2*>(ws + L.gate);
    if (has_ve) {
        const int gblocks = (int)std::min<long long>((M + 127) / 128, 148ll * 16);
        const int wg_smem = 32 * s.Hkv * (int)sizeof(double) <= 48 * 1024;
        swa::gate_kernel<<<gblocks, 128, wg_smem ? 32 * s.Hkv * sizeof(double) : 0, st>>>(
            static_cast<const bf*>(x), static_cast<const bf*>(Wg), gate, (int)M, s.Hkv, C, wg_smem);
    }
    const int N = (s.H + 2 * s.Hkv) * s.D;
    const int BN = ((s.H * s.D) % 256 == 0 && (s.Hkv * s.D) % 256 == 0) ? 256 : 128;
    CUtensorMap tx, tw;
    if (!make_matrix_map(&tx, x, M, C, 128) || !make_matrix_map(&tw, Wqkv, N, C, BN)) return SWA_ERR_CUDA;
    swa::QkvParams p{};
    p.M = (int)M;
    p.T = s.T;
    p.C = C;
    p.H = s.H;
    p.Hkv = s.Hkv;
    p.N = N;
    p.n_ntiles = (N + BN - 1) / BN;
    p.n_tiles = (int)((M + 127) / 128) * p.n_ntiles;
    p.eps = eps;
    p.tab2 = reinterpret_cast<const float2*>(ws + L.tab64);
    p.gate = has_ve ? gate : nullptr;
    p.ve = static_cast<const bf*>(ve);
    p.qh = static_cast<bf*>(qh);
    p.kh = static_cast<bf*>(kh);
    p.vp = static_cast<bf*>(vp);
    p.sched_zero = sched_zero;
    p.wait_limit_ns = wait_limit_ns();
    const dim3 grid((unsigned)std::min(p.n_tiles, g_num_sms[dev]));
#define SWA_QKV(DD, BB, VE) \
    swa::qkv_gemm_kernel<DD, BB, VE><<<grid, swa::QkvCfg<BB>::THREADS, swa::QkvCfg<BB>::SMEM_TOTAL, st>>>(tx, tw, p)
    if (s.D == 128) {
        if (BN == 256) { if (has_ve) SWA_QKV(128, 256, true); else SWA_QKV(128, 256, false); }
        else { if (has_ve) SWA_QKV(128, 128, true); else SWA_QKV(128, 128, false); }
    } else {
        if (BN == 256) { if (has_ve) SWA_QKV(64, 256, true); else SWA_QKV(64, 256, false); }
        else { if (has_ve) SWA_QKV(64, 128, true); else SWA_QKV(64, 128, false); }
    }
#undef SWA_QKV
    return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

// ---------------------------------------------------------------------------- backward

// The forward's sections (qhat, khat, v', gate, RoPE tables, counters; the prologue rewrites them)
// followed by the backward's: row statistics (B, H, Tp) float2 | dqhat (B,T,H,D) fp32 |
// dkhat, dv' (B,T,Hkv,D) fp32 | dz (B,T,Hkv) fp32 and the dWg partial sums (value-embedding
// layers only).  The backward kernels' scheduler counters are ints 4..7 of the counter section.
struct BwdLayout {
    WsLayout f;
    size_t rowstat, dz, wgp, dstart, dend, total;
    int Tp, wg_blocks, wg_rows;
};

BwdLayout bwd_layout(const Shape& s, bool has_ve) {
    BwdLayout w{};
    w.f = ws_layout(s, has_ve);
    w.Tp = ((s.T + 127) / 128) * 128;
    const long long n_bt = (long long)s.B * s.T;
    w.wg_rows = 32;
    w.wg_blocks = has_ve ? (int)((n_bt + w.wg_rows - 1) / w.wg_rows) : 0;
    size_t o = w.f.total;
    w.rowstat = o;
    o += round_up((size_t)s.B * s.H * w.Tp * sizeof(float2));
    w.dz = o;
    o += has_ve ? round_up((size_t)n_bt * s.Hkv * 4) : 0;
    w.wgp = o;
    o += has_ve ? round_up((size_t)w.wg_blocks * 32 * s.Hkv * 4) : 0;
    // document starts and ends (document-masked calls; a few bytes per position, always reserved)
    w.dstart = o;
    o += round_up((size_t)n_bt * 4);
    w.dend = o;
    o += round_up((size_t)n_bt * 4);
    w.total = o;
    return w;
}

// A second stream per device for kernels of one call that do not depend on the kernels before
// them on the caller's stream: they are forked from the caller's stream (an event recorded there,
// waited on here) and joined back the same way, so everything the caller enqueued earlier happens
// before them and everything after the join happens after them.  Calls that share the side stream
// serialise their side kernels on it.
std::mutex g_side_mu;                 // guards the creation of the side streams
std::mutex g_side_mu_call[64];        // held by a call while it uses its device's side stream
cudaStream_t g_side[64] = {nullptr};

// `to` waits for everything enqueued on `from` so far.  The event is released at once; CUDA keeps
// it until the wait is resolved.
int stream_wait(cudaStream_t to, cudaStream_t from) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        return SWA_ERR_CUDA;
    }
    const bool ok = cudaEventRecord(e, from) == cudaSuccess && cudaStreamWaitEvent(to, e, 0) == cudaSuccess;
    cudaEventDestroy(e);
    if (!ok) {
        cudaGetLastError();
        return SWA_ERR_CUDA;
    }
    return SWA_OK;
}

int side_stream(int dev, cudaStream_t* out) {
    std::lock_guard<std::mutex> lk(g_side_mu);
    if (g_side[dev] == nullptr && cudaStreamCreateWithFlags(&g_side[dev], cudaStreamNonBlocking) != cudaSuccess) {
        cudaGetLastError();
        g_side[dev] = nullptr;
        return SWA_ERR_CUDA;
    }
    *out = g_side[dev];
    return SWA_OK;
}

int launch_backward(int dev, const void* q, const void* k, const void* v, const void* ve,
                    const void* gate_x, const void* Wg, const void* out, const float* lse,
                    const void* dout, const float* dlse, void* dq, void* dk, void* dv, void* dve,
                    float* dgate_x, float* dWg, const Shape& s, int window, float rope_base, float eps,
                    uint8_t* ws, const BwdLayout& L, cudaStream_t st, const int* doc = nullptr,
                    bool prologue_saved = false) {
    using bf = __nv_bfloat16;
    const bool has_ve = ve != nullptr;
    int rc;
    // The row statistics need only out, dout, lse and dlse: they run on the side stream while the
    // caller's stream recomputes the prologue, and the tensor-core kernels wait for both.  The
    // side stream is held for the whole call, so that its kernels are this call's alone.
    std::lock_guard<std::mutex> side_lk(g_side_mu_call[dev]);
    cudaStream_t side = nullptr;
    if ((rc = side_stream(dev, &side)) != SWA_OK) return rc;
    if ((rc = stream_wait(side, st)) != SWA_OK) return rc;
    int* sched4 = reinterpret_cast<int*>(ws + L.f.sched) + 4;
    float2* rowstat = reinterpret_cast<float2*>(ws + L.rowstat);
    {
        const long long rows = (long long)s.B * s.H * L.Tp;
        const int blocks = (int)((rows * (s.D / 8) + 255) / 256);   // D / 8 lanes per row
        if (s.D == 128)
            swa::bwd_rowstat_kernel<128><<<blocks, 256, 0, side>>>(static_cast<const bf*>(out), static_cast<const bf*>(dout),
                                                                   lse, dlse, rowstat, s.B, s.T, s.H, L.Tp, sched4);
        else
            swa::bwd_rowstat_kernel<64><<<blocks, 256, 0, side>>>(static_cast<const bf*>(out), static_cast<const bf*>(dout),
                                                                  lse, dlse, rowstat, s.B, s.T, s.H, L.Tp, sched4);
        if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
    }
    // qhat, khat, v' and the gate exactly as the forward computed them (unless the caller's forward
    // left them in this workspace).
    if (!prologue_saved) {
        if ((rc = launch_rope_table(ws, L.f, s, rope_base, st)) != SWA_OK) return rc;
        if ((rc = launch_prologue(q, k, v, ve, gate_x, Wg, ws, L.f, s, eps, st)) != SWA_OK) return rc;
    }
    if ((rc = stream_wait(st, side)) != SWA_OK) return rc;

    CUtensorMap tq, tk, tv, tdo;
    const void* vsrc = has_ve ? static_cast<const void*>(ws + L.f.vp) : v;
    if (!make_tile_map(&tq, ws + L.f.qh, s, s.H) || !make_tile_map(&tk, ws + L.f.kh, s, s.Hkv) ||
        !make_tile_map(&tv, vsrc, s, s.Hkv) || !make_tile_map(&tdo, dout, s, s.H))
        return SWA_ERR_CUDA;
    swa::BwdParams p{};
    p.B = s.B;
    p.T = s.T;
    p.H = s.H;
    p.Hkv = s.Hkv;
    p.G = s.H / s.Hkv;
    p.W = (window <= 0 || window >= s.T) ? s.T : window;
    p.n_tiles = (s.T + 127) / 128;
    p.Tp = L.Tp;
    p.c1 = (float)(1.4426950408889634 / std::sqrt((double)s.D));
    p.inv_sqrt_d = (float)(1.0 / std::sqrt((double)s.D));
    p.rowstat = rowstat;
    p.xq = static_cast<const bf*>(q);
    p.xk = static_cast<const bf*>(k);
    p.ve = static_cast<const bf*>(ve);
    p.gate = has_ve ? reinterpret_cast<const float2*>(ws + L.f.gate) : nullptr;
    p.rope_base = (double)rope_base;
    p.eps = eps;
    p.dq = static_cast<bf*>(dq);
    p.dk = static_cast<bf*>(dk);
    p.dv = static_cast<bf*>(dv);
    p.dve = static_cast<bf*>(dve);
    p.dz = has_ve ? reinterpret_cast<float*>(ws + L.dz) : nullptr;
    p.wait_limit_ns = wait_limit_ns();
    if (doc) {
        p.dstart = reinterpret_cast<int*>(ws + L.dstart);
        p.dend = reinterpret_cast<int*>(ws + L.dend);
        swa::doc_start_kernel<<<s.B, 1024, 0, st>>>(doc, reinterpret_cast<int*>(ws + L.dstart),
                                                   reinterpret_cast<int*>(ws + L.dend), s.T);
    }
    const long long slice_bytes = 4ll * s.T * s.D;   // two bf16 (T, D) slices
    // Query tiles: chunks of (b, h) slices whose K and V' fit in ~40 MB of L2.
    swa::BwdParams pq = p;
    pq.n_items = p.n_tiles * s.H * s.B;
    pq.chunk_bh = (int)std::max<long long>(1, std::min<long long>((40ll << 20) / slice_bytes, (long long)s.B * s.H));
    pq.sched = sched4;
    // Key tiles: chunks of (b, hk) slices whose G query heads of Q and dO fit likewise.
    swa::BwdParams pk = p;
    pk.n_items = p.n_tiles * s.Hkv * s.B;
    pk.chunk_bh = (int)std::max<long long>(
        1, std::min<long long>((40ll << 20) / (slice_bytes * p.G), (long long)s.B * s.Hkv));
    pk.sched = sched4 + 2;
    const dim3 gq((unsigned)std::min(pq.n_items, g_num_sms[dev]));
    const dim3 gk((unsigned)std::min(pk.n_items, g_num_sms[dev]));
#define SWA_BWD_TC(DD, DC)                                                                                  \
    do {                                                                                                    \
        using C = swa::BwdCfg<DD>;                                                                          \
        swa::attn_bwd_dq_kernel<DD, DC><<<gq, C::THREADS, C::DQ_SMEM, st>>>(tq, tk, tv, tdo, pq);            \
        swa::attn_bwd_dkv_kernel<DD, DC><<<gk, C::THREADS, C::KV_SMEM, st>>>(tq, tk, tv, tdo, pk);           \
    } while (0)
    if (s.D == 128) {
        if (doc) SWA_BWD_TC(128, true); else SWA_BWD_TC(128, false);
    } else {
        if (doc) SWA_BWD_TC(64, true); else SWA_BWD_TC(64, false);
    }
#undef SWA_BWD_TC

    // The rest of the prologue in reverse: the gate's inputs from dz (the epilogues did the rows).
    float* dz = reinterpret_cast<float*>(ws + L.dz);
    if (has_ve) {
        // dgate_x on the caller's stream, dWg (two steps) on the side stream; both only read dz.
        if ((rc = stream_wait(side, st)) != SWA_OK) return rc;
        const long long n_bt = (long long)s.B * s.T;
        const int bgx = (int)std::min<long long>((n_bt * 32 + 255) / 256, 148ll * 16);
        swa::bwd_gate_x_kernel<<<bgx, 256, 0, st>>>(dz, static_cast<const bf*>(Wg), dgate_x, n_bt, s.Hkv);
        float* part = reinterpret_cast<float*>(ws + L.wgp);
        swa::bwd_wg_partial_kernel<<<L.wg_blocks, 256, 0, side>>>(dz, static_cast<const bf*>(gate_x), part, n_bt,
                                                                  s.Hkv, L.wg_rows);
        const int n = 32 * s.Hkv;
        swa::bwd_wg_final_kernel<<<n, 256, 0, side>>>(part, dWg, L.wg_blocks, n);
        if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
        if ((rc = stream_wait(st, side)) != SWA_OK) return rc;
    }
    return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

// ------------------------------------------------------------- library-owned workspace

struct DevCache {
    void* ptr = nullptr;
    size_t bytes = 0;
    int tab_T = -1, tab_D = -1;
    float tab_base = 0.f;
    size_t tab_off = (size_t)-1;
    cudaEvent_t last_use = nullptr;       // recorded after the last call's launches
    cudaStream_t last_stream = nullptr;   // the stream of that call
};
DevCache g_cache[64];

}  // namespace

extern "C" {

int swa_attn_version(void) { return kVersion; }

const char* swa_attn_strerror(int status) {
    switch (status) {
        case SWA_OK: return "ok";
        case SWA_ERR_INVALID_ARG: return "invalid argument";
        case SWA_ERR_UNSUPPORTED: return "unsupported size, head dim or device";
        case SWA_ERR_MISALIGNED: return "pointer not aligned (tensors and workspace need 16 bytes)";
        case SWA_ERR_CUDA: return "CUDA call failed";
        case SWA_ERR_TIMEOUT: return "a bounded wait inside a kernel expired";
        case SWA_ERR_NO_MEMORY: return "workspace too small or allocation failed";
        case SWA_ERR_NO_DEVICE: return "no CUDA device";
        default: return "unknown status";
    }
}

int swa_attn_set_wait_limit_ms(int ms) {
    const unsigned long long prev = wait_limit_ns();
    if (ms >= 1) g_wait_limit_ns.store((unsigned long long)ms * 1000000ull);
    return (int)(prev / 1000000ull);
}

size_t swa_attn_workspace_offset(int B, int T, int H, int D, int has_ve, int section) {
    Shape s;
    if (check_sizes(B, T, H, D, &s) != SWA_OK) return (size_t)-1;
    const WsLayout L = ws_layout(s, has_ve != 0);
    switch (section) {
        case SWA_WS_QHAT: return L.qh;
        case SWA_WS_KHAT: return L.kh;
        case SWA_WS_VPRIME: return has_ve ? L.vp : (size_t)-1;
        case SWA_WS_ROPE_TABLE: return L.tab32;
        default: return (size_t)-1;
    }
}

size_t swa_attn_workspace_bytes(int B, int T, int H, int D, int has_ve) {
    Shape s;
    if (check_sizes(B, T, H, D, &s) != SWA_OK) return 0;
    return ws_layout(s, has_ve != 0).total;
}

int swa_attn_rope_table(int B, int T, int H, int D, int has_ve, float rope_base, void* workspace,
                        size_t ws_bytes, swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc != SWA_OK) return rc;
    if (!std::isfinite(rope_base) || !(rope_base > 0.f) || !workspace) return SWA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SWA_ERR_MISALIGNED;
    const WsLayout L = ws_layout(s, has_ve != 0);
    if (ws_bytes < L.total) return SWA_ERR_NO_MEMORY;
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    return launch_rope_table(static_cast<uint8_t*>(workspace), L, s, rope_base,
                             reinterpret_cast<cudaStream_t>(stream));
}

int swa_attn_prologue(const void* q, const void* k, const void* v, const void* ve,
                      const void* gate_x, const void* Wg, int B, int T, int H, int D,
                      float rope_base, float eps, void* workspace, size_t ws_bytes,
                      swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc == SWA_OK) rc = check_layer_args(q, k, v, ve, gate_x, Wg, rope_base, eps);
    if (rc != SWA_OK) return rc;
    if (!workspace) return SWA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SWA_ERR_MISALIGNED;
    const WsLayout L = ws_layout(s, ve != nullptr);
    if (ws_bytes < L.total) return SWA_ERR_NO_MEMORY;
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    return launch_prologue(q, k, v, ve, gate_x, Wg, static_cast<uint8_t*>(workspace), L, s, eps,
                           reinterpret_cast<cudaStream_t>(stream));
}

int swa_attn_attention(const void* v, int has_ve, void* out, float* lse, int B, int T, int H, int D,
                       int window, void* workspace, size_t ws_bytes, swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc != SWA_OK) return rc;
    if (!workspace || (!has_ve && !v)) return SWA_ERR_INVALID_ARG;
    if ((rc = check_outputs(out, lse)) != SWA_OK) return rc;
    if (!aligned(workspace, 16) || (!has_ve && !aligned(v, 16))) return SWA_ERR_MISALIGNED;
    const WsLayout L = ws_layout(s, has_ve != 0);
    if (ws_bytes < L.total) return SWA_ERR_NO_MEMORY;
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    return launch_attention(dev, v, has_ve != 0, out, lse, s, window, static_cast<uint8_t*>(workspace), L,
                            reinterpret_cast<cudaStream_t>(stream));
}

int swa_attn_fwd_ws(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                    const void* Wg, void* out, float* lse, int B, int T, int H, int D, int window,
                    float rope_base, float eps, void* workspace, size_t ws_bytes,
                    swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc == SWA_OK) rc = check_layer_args(q, k, v, ve, gate_x, Wg, rope_base, eps);
    if (rc == SWA_OK) rc = check_outputs(out, lse);
    if (rc != SWA_OK) return rc;
    rc = swa_attn_rope_table(B, T, H, D, ve != nullptr, rope_base, workspace, ws_bytes, stream);
    if (rc != SWA_OK) return rc;
    rc = swa_attn_prologue(q, k, v, ve, gate_x, Wg, B, T, H, D, rope_base, eps, workspace, ws_bytes, stream);
    if (rc != SWA_OK) return rc;
    return swa_attn_attention(v, ve != nullptr, out, lse, B, T, H, D, window, workspace, ws_bytes, stream);
}

}  // extern "C"

namespace {

// The forward with the library-owned workspace of the current device (validated arguments).
int fwd_library_ws(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                   const void* Wg, const int* doc, void* out, float* lse, const Shape& s, int window,
                   float rope_base, float eps, swa_stream_t stream) {
    int rc;
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    const int T = s.T, D = s.D;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool has_ve = ve != nullptr;
    const WsLayout L = ws_layout(s, has_ve, doc != nullptr);

    const unsigned long long limit = wait_limit_ns();   // read before taking the cache lock
    (void)limit;
    std::lock_guard<std::mutex> lk(g_cache_mu);
    DevCache& c = g_cache[dev];
    // The cached workspace (and its RoPE table) may still be in use by the previous call's kernels
    // on another stream: this stream waits for them before it touches, reuses or frees it.
    if (c.last_use != nullptr && c.last_stream != st) {
        if (cudaStreamWaitEvent(st, c.last_use, 0) != cudaSuccess) {
            cudaGetLastError();
            return SWA_ERR_CUDA;
        }
    }
    if (c.last_use == nullptr &&
        cudaEventCreateWithFlags(&c.last_use, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        c.last_use = nullptr;
        return SWA_ERR_CUDA;
    }
    if (c.bytes < L.total) {
        if (c.ptr) cudaFreeAsync(c.ptr, st);
        c.ptr = nullptr;
        c.bytes = 0;
        c.tab_T = -1;
        void* p = nullptr;
        if (cudaMallocAsync(&p, L.total, st) != cudaSuccess) {
            cudaGetLastError();
            return SWA_ERR_NO_MEMORY;
        }
        c.ptr = p;
        c.bytes = L.total;
    }
    uint8_t* ws = static_cast<uint8_t*>(c.ptr);
    if (c.tab_T != T || c.tab_D != D || c.tab_base != rope_base || c.tab_off != L.tab32) {
        if ((rc = launch_rope_table(ws, L, s, rope_base, st)) != SWA_OK) return rc;
        c.tab_T = T;
        c.tab_D = D;
        c.tab_base = rope_base;
        c.tab_off = L.tab32;
    }
    int* dstart = doc ? reinterpret_cast<int*>(ws + L.dstart) : nullptr;
    if (doc) {
        swa::doc_start_kernel<<<s.B, 1024, 0, st>>>(doc, dstart, nullptr, s.T);
        rc = cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
    } else {
        rc = SWA_OK;
    }
    if (rc == SWA_OK) rc = launch_prologue(q, k, v, ve, gate_x, Wg, ws, L, s, eps, st);
    if (rc == SWA_OK) rc = launch_attention(dev, v, has_ve, out, lse, s, window, ws, L, st, dstart);
    // Recorded after whatever was enqueued, also on failure, so the next call orders after it.
    if (cudaEventRecord(c.last_use, st) != cudaSuccess) {
        cudaGetLastError();
        if (rc == SWA_OK) rc = SWA_ERR_CUDA;
    }
    c.last_stream = st;
    return rc;
}

}  // namespace

// The caches (B, Tmax, Hkv, D) bf16 as 3-D {D, Hkv, B * Tmax}; box = D features x 1 head x KB
// positions, no swizzle.  Positions past B * Tmax read as zeros.
bool make_cache_map(CUtensorMap* m, const void* base, int B, int Tmax, int Hkv, int D, int kb) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)B * Tmax};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
    const cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)kb};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Attention of the new tokens over the window keys [lo, lo + n_keys): a cluster of n_chunks CTAs
// per row b*H + h.  n_chunks (at most 8, the portable cluster size) is the number of the GPU's
// resident CTA slots per row, so that one wave streams the whole window; each CTA takes whole
// KB-key tiles.
template <int D>
int launch_decode_attention_d(int dev, const void* q, const void* k_cache, const void* v_cache, const int* doc_start,
                              void* out, float* lse, int B, int Tmax, int H, int Hkv, int lo, int n_keys, int pos,
                              double rope_base, double eps, cudaStream_t st) {
    using C = swa::DecCfg<D>;
    CUtensorMap tk, tv;
    if (!make_cache_map(&tk, k_cache, B, Tmax, Hkv, D, C::KB) || !make_cache_map(&tv, v_cache, B, Tmax, Hkv, D, C::KB))
        return SWA_ERR_CUDA;
    // resident CTAs per SM, found once per device (threads that race here store the same value)
    static std::atomic<int> per_sm[64];
    int n_per_sm = per_sm[dev].load(std::memory_order_relaxed);
    if (n_per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n_per_sm, swa::decode_attn_kernel<D>, C::THREADS,
                                                          C::SMEM) != cudaSuccess || n_per_sm < 1) {
            cudaGetLastError();
            n_per_sm = 1;
        }
        per_sm[dev].store(n_per_sm, std::memory_order_relaxed);
    }
    const long long rows = (long long)B * H;
    const long long slots = (long long)n_per_sm * g_num_sms[dev];
    const int n_tiles = (n_keys + C::KB - 1) / C::KB;
    int n_chunks = (int)std::max<long long>(1, std::min<long long>(slots / rows, swa::kDecodeMaxCluster));
    n_chunks = std::min(n_chunks, n_tiles);
    const int tiles_per_chunk = (n_tiles + n_chunks - 1) / n_chunks;
    n_chunks = (n_tiles + tiles_per_chunk - 1) / tiles_per_chunk;
    swa::DecParams p{};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.rope_base = rope_base;
    p.eps = eps;
    p.pos = pos;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.doc_start = doc_start;
    p.H = H;
    p.Hkv = Hkv;
    p.Tmax = Tmax;
    p.lo = lo;
    p.n_keys = n_keys;
    p.tiles_per_chunk = tiles_per_chunk;
    const double log2e = 1.4426950408889634;
    const double m0 = std::sqrt((double)D) * (1.0 + 1.0 / 64.0);
    p.c1 = (float)(log2e / std::sqrt((double)D));
    p.c2 = (float)(m0 * log2e);
    p.m0 = (float)m0;
    p.wait_limit_ns = wait_limit_ns();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * n_chunks));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)n_chunks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // may start before the prologue kernel ends (the kernel waits where it reads that kernel's output)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, swa::decode_attn_kernel<D>, tk, tv, p) != cudaSuccess) return SWA_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int launch_decode_attention(int dev, const void* q, const void* k_cache, const void* v_cache, const int* doc_start,
                            void* out, float* lse, int B, int Tmax, int H, int Hkv, int D, int lo, int n_keys, int pos,
                            double rope_base, double eps, cudaStream_t st) {
    return D == 128 ? launch_decode_attention_d<128>(dev, q, k_cache, v_cache, doc_start, out, lse, B, Tmax, H, Hkv,
                                                     lo, n_keys, pos, rope_base, eps, st)
                    : launch_decode_attention_d<64>(dev, q, k_cache, v_cache, doc_start, out, lse, B, Tmax, H, Hkv,
                                                    lo, n_keys, pos, rope_base, eps, st);
}

extern "C" {

int swa_attn_fwd_gqa(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                     const void* Wg, void* out, float* lse, int B, int T, int H, int Hkv, int D,
                     int window, float rope_base, float eps, swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc == SWA_OK) rc = check_kv_heads(Hkv, &s);
    if (rc == SWA_OK) rc = check_layer_args(q, k, v, ve, gate_x, Wg, rope_base, eps);
    if (rc == SWA_OK) rc = check_outputs(out, lse);
    if (rc != SWA_OK) return rc;
    return fwd_library_ws(q, k, v, ve, gate_x, Wg, nullptr, out, lse, s, window, rope_base, eps, stream);
}

int swa_attn_fwd_doc(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                     const void* Wg, const int* doc, void* out, float* lse, int B, int T, int H, int Hkv,
                     int D, int window, float rope_base, float eps, swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc == SWA_OK) rc = check_kv_heads(Hkv, &s);
    if (rc == SWA_OK) rc = check_layer_args(q, k, v, ve, gate_x, Wg, rope_base, eps);
    if (rc == SWA_OK) rc = check_outputs(out, lse);
    if (rc != SWA_OK) return rc;
    if (!doc) return SWA_ERR_INVALID_ARG;
    if (!aligned(doc, 4)) return SWA_ERR_MISALIGNED;
    return fwd_library_ws(q, k, v, ve, gate_x, Wg, doc, out, lse, s, window, rope_base, eps, stream);
}

int swa_attn_fwd(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                 const void* Wg, void* out, float* lse, int B, int T, int H, int D, int window,
                 float rope_base, float eps, swa_stream_t stream) {
    return swa_attn_fwd_gqa(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, H, D, window, rope_base, eps,
                            stream);
}

// --------------------------------------------------------------- fused q/k/v projection

size_t swa_attn_fwd_x_workspace_bytes(int B, int T, int H, int Hkv, int D) {
    Shape s;
    if (check_sizes(B, T, H, D, &s) != SWA_OK || check_kv_heads(Hkv, &s) != SWA_OK) return 0;
    return ws_layout(s, true).total;   // v' always lives in the workspace on this path
}

int swa_attn_qkv_prologue(const void* x, const void* Wqkv, const void* ve, const void* Wg, void* qh, void* kh,
                          void* vp, int B, int T, int C, int H, int Hkv, int D, float rope_base, float eps,
                          void* workspace, size_t ws_bytes, swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc == SWA_OK) rc = check_kv_heads(Hkv, &s);
    if (rc == SWA_OK) rc = check_qkv_args(x, Wqkv, ve, Wg, s, C, rope_base, eps);
    if (rc != SWA_OK) return rc;
    if (!qh || !kh || !vp || !workspace) return SWA_ERR_INVALID_ARG;
    if (!aligned(qh, 16) || !aligned(kh, 16) || !aligned(vp, 16) || !aligned(workspace, 16)) return SWA_ERR_MISALIGNED;
    const WsLayout L = ws_layout(s, true);
    if (ws_bytes < L.total) return SWA_ERR_NO_MEMORY;
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if ((rc = launch_rope_table(ws, L, s, rope_base, st, true)) != SWA_OK) return rc;
    return launch_qkv(dev, x, Wqkv, ve, Wg, C, s, eps, ws, L, qh, kh, vp, nullptr, st);
}

int swa_attn_fwd_x(const void* x, const void* Wqkv, const void* ve, const void* Wg, void* out, float* lse, int B,
                   int T, int C, int H, int Hkv, int D, int window, float rope_base, float eps, void* workspace,
                   size_t ws_bytes, swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc == SWA_OK) rc = check_kv_heads(Hkv, &s);
    if (rc == SWA_OK) rc = check_qkv_args(x, Wqkv, ve, Wg, s, C, rope_base, eps);
    if (rc == SWA_OK) rc = check_outputs(out, lse);
    if (rc != SWA_OK) return rc;
    if (!workspace) return SWA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SWA_ERR_MISALIGNED;
    const WsLayout L = ws_layout(s, true);
    if (ws_bytes < L.total) return SWA_ERR_NO_MEMORY;
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if ((rc = launch_rope_table(ws, L, s, rope_base, st, true)) != SWA_OK) return rc;
    if ((rc = launch_qkv(dev, x, Wqkv, ve, Wg, C, s, eps, ws, L, ws + L.qh, ws + L.kh, ws + L.vp,
                         reinterpret_cast<int*>(ws + L.sched), st)) != SWA_OK)
        return rc;
    return launch_attention(dev, nullptr, true, out, lse, s, window, ws, L, st);
}

// ---------------------------------------------------------------------------- backward

size_t swa_attn_bwd_workspace_bytes(int B, int T, int H, int Hkv, int D, int has_ve) {
    Shape s;
    if (check_sizes(B, T, H, D, &s) != SWA_OK || check_kv_heads(Hkv, &s) != SWA_OK) return 0;
    return bwd_layout(s, has_ve != 0).total;
}

}  // extern "C"

namespace {

// The backward entry points after argument checks; prologue_saved: qhat, khat, v', the gates and
// the RoPE tables are already in the workspace (left there by swa_attn_fwd_ws).
int bwd_checked(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                const void* Wg, const int* doc, const void* out, const float* lse, const void* dout,
                const float* dlse, void* dq, void* dk, void* dv, void* dve, float* dgate_x,
                float* dWg, int B, int T, int H, int Hkv, int D, int window, float rope_base,
                float eps, void* workspace, size_t ws_bytes, swa_stream_t stream, bool prologue_saved) {
    if (doc != nullptr && !aligned(doc, 4)) return SWA_ERR_MISALIGNED;
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc == SWA_OK) rc = check_kv_heads(Hkv, &s);
    if (rc == SWA_OK) rc = check_layer_args(q, k, v, ve, gate_x, Wg, rope_base, eps);
    if (rc != SWA_OK) return rc;
    const bool has_ve = ve != nullptr;
    if (!out || !lse || !dout || !dq || !dk || !dv || !workspace) return SWA_ERR_INVALID_ARG;
    const int n_vegrad = (dve != nullptr) + (dgate_x != nullptr) + (dWg != nullptr);
    if (n_vegrad != (has_ve ? 3 : 0)) return SWA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4) || (dlse && !aligned(dlse, 4)) || !aligned(workspace, 16))
        return SWA_ERR_MISALIGNED;
    if (has_ve && (!aligned(dve, 16) || !aligned(dgate_x, 4) || !aligned(dWg, 4))) return SWA_ERR_MISALIGNED;
    const BwdLayout L = bwd_layout(s, has_ve);
    if (ws_bytes < L.total) return SWA_ERR_NO_MEMORY;
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    return launch_backward(dev, q, k, v, ve, gate_x, Wg, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg, s,
                           window, rope_base, eps, static_cast<uint8_t*>(workspace), L,
                           reinterpret_cast<cudaStream_t>(stream), doc, prologue_saved);
}

}  // namespace

extern "C" {

int swa_attn_bwd_doc(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                     const void* Wg, const int* doc, const void* out, const float* lse, const void* dout,
                     const float* dlse, void* dq, void* dk, void* dv, void* dve, float* dgate_x,
                     float* dWg, int B, int T, int H, int Hkv, int D, int window, float rope_base,
                     float eps, void* workspace, size_t ws_bytes, swa_stream_t stream) {
    return bwd_checked(q, k, v, ve, gate_x, Wg, doc, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg, B, T, H,
                       Hkv, D, window, rope_base, eps, workspace, ws_bytes, stream, false);
}

int swa_attn_bwd_saved(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                       const void* Wg, const void* out, const float* lse, const void* dout, const float* dlse,
                       void* dq, void* dk, void* dv, void* dve, float* dgate_x, float* dWg, int B, int T,
                       int H, int D, int window, float rope_base, float eps, void* workspace, size_t ws_bytes,
                       swa_stream_t stream) {
    return bwd_checked(q, k, v, ve, gate_x, Wg, nullptr, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg, B, T,
                       H, H, D, window, rope_base, eps, workspace, ws_bytes, stream, true);
}

int swa_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                     const void* Wg, const void* out, const float* lse, const void* dout,
                     const float* dlse, void* dq, void* dk, void* dv, void* dve, float* dgate_x,
                     float* dWg, int B, int T, int H, int Hkv, int D, int window, float rope_base,
                     float eps, void* workspace, size_t ws_bytes, swa_stream_t stream) {
    return swa_attn_bwd_doc(q, k, v, ve, gate_x, Wg, nullptr, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x,
                            dWg, B, T, H, Hkv, D, window, rope_base, eps, workspace, ws_bytes, stream);
}

int swa_attn_bwd(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                 const void* Wg, const void* out, const float* lse, const void* dout, const float* dlse,
                 void* dq, void* dk, void* dv, void* dve, float* dgate_x, float* dWg, int B, int T, int H,
                 int D, int window, float rope_base, float eps, void* workspace, size_t ws_bytes,
                 swa_stream_t stream) {
    return swa_attn_bwd_gqa(q, k, v, ve, gate_x, Wg, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg, B, T,
                            H, H, D, window, rope_base, eps, workspace, ws_bytes, stream);
}

// ------------------------------------------------------------- decode step with a KV cache
//
// Workspace: qhat of the new token (B*H*D bf16), 1024-byte aligned.  The chunks of a row are
// combined inside their cluster, so nothing else is stored.

size_t swa_attn_decode_workspace_bytes(int B, int Tmax, int H, int D, int has_ve, int window) {
    Shape s;
    if (check_sizes(B, Tmax, H, D, &s) != SWA_OK) return 0;
    (void)has_ve;
    (void)window;
    return round_up((size_t)B * H * D * 2);
}

int swa_attn_decode_doc(const void* q, const void* k, const void* v, const void* ve,
                        const void* gate_x, const void* Wg, void* k_cache, void* v_cache, int pos,
                        const int* doc_start, void* out, float* lse, int B, int Tmax, int H, int Hkv,
                        int D, int window, float rope_base, float eps, void* workspace, size_t ws_bytes,
                        swa_stream_t stream) {
    if (doc_start != nullptr && !aligned(doc_start, 4)) return SWA_ERR_MISALIGNED;
    Shape s;
    int rc = check_sizes(B, Tmax, H, D, &s);
    if (rc == SWA_OK) rc = check_kv_heads(Hkv, &s);
    if (rc == SWA_OK) rc = check_layer_args(q, k, v, ve, gate_x, Wg, rope_base, eps);
    if (rc == SWA_OK) rc = check_outputs(out, lse);
    if (rc != SWA_OK) return rc;
    if (pos < 0 || pos >= Tmax || !k_cache || !v_cache || !workspace) return SWA_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(workspace, 16)) return SWA_ERR_MISALIGNED;
    const bool has_ve = ve != nullptr;
    if (ws_bytes < swa_attn_decode_workspace_bytes(B, Tmax, H, D, has_ve, window)) return SWA_ERR_NO_MEMORY;
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    using bf = __nv_bfloat16;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    bf* qh = reinterpret_cast<bf*>(ws);   // unused by the key/value pass (qhat is formed by the attention kernel)
    {
        const int rows_per_block = 256 / (D / 8);
        const bf* qp = static_cast<const bf*>(q);
        const bf* kp = static_cast<const bf*>(k);
        const bf* vp = static_cast<const bf*>(v);
        const bf* vep = static_cast<const bf*>(ve);
        const bf* gx = static_cast<const bf*>(gate_x);
        const bf* wg = static_cast<const bf*>(Wg);
        bf* kc = static_cast<bf*>(k_cache);
        bf* vc = static_cast<bf*>(v_cache);
        const double base = (double)rope_base, e = (double)eps;
        const int kv_rows = B * Hkv;
        const int kv_blocks = std::max(1, std::min((kv_rows + rows_per_block - 1) / rows_per_block, 148 * 8));
    // The token prologue writes khat and v' to the caches; the attention kernel forms qhat itself.
#define SWA_DEC_PRO(DD, VE)                                                                               \
    swa::decode_prologue_kernel<DD, VE, 2><<<kv_blocks, 256, 0, st>>>(qp, kp, vp, vep, gx, wg, qh, kc, vc,     \
                                                                      kv_rows, Hkv, Tmax, pos, base, e)
        if (D == 128) {
            if (has_ve)
                SWA_DEC_PRO(128, true);
            else
                SWA_DEC_PRO(128, false);
        } else {
            if (has_ve)
                SWA_DEC_PRO(64, true);
            else
                SWA_DEC_PRO(64, false);
        }
#undef SWA_DEC_PRO
    }
    const int W = (window <= 0 || window >= Tmax) ? Tmax : window;
    const int lo = std::max(0, pos - W + 1);
    const int n_keys = pos - lo + 1;
    return launch_decode_attention(dev, q, k_cache, v_cache, doc_start, out, lse, B, Tmax, H, Hkv, D, lo, n_keys, pos,
                                   (double)rope_base, (double)eps, st);
}

int swa_attn_decode_gqa(const void* q, const void* k, const void* v, const void* ve,
                        const void* gate_x, const void* Wg, void* k_cache, void* v_cache, int pos,
                        void* out, float* lse, int B, int Tmax, int H, int Hkv, int D, int window,
                        float rope_base, float eps, void* workspace, size_t ws_bytes,
                        swa_stream_t stream) {
    return swa_attn_decode_doc(q, k, v, ve, gate_x, Wg, k_cache, v_cache, pos, nullptr, out, lse, B, Tmax, H, Hkv,
                               D, window, rope_base, eps, workspace, ws_bytes, stream);
}

int swa_attn_decode(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                    const void* Wg, void* k_cache, void* v_cache, int pos, void* out, float* lse,
                    int B, int Tmax, int H, int D, int window, float rope_base, float eps,
                    void* workspace, size_t ws_bytes, swa_stream_t stream) {
    return swa_attn_decode_gqa(q, k, v, ve, gate_x, Wg, k_cache, v_cache, pos, out, lse, B, Tmax, H, H, D,
                               window, rope_base, eps, workspace, ws_bytes, stream);
}

int swa_attn_selftest_wait(int limit_ms, swa_stream_t stream) {
    if (limit_ms < 1 || limit_ms > 10000) return SWA_ERR_INVALID_ARG;
    int dev;
    int rc = device_ready(&dev);
    if (rc != SWA_OK) return rc;
    swa::wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_ms * 1000000ull);
    return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_attn_last_device_status(swa_stream_t stream, unsigned int* detail) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return SWA_ERR_CUDA;
    }
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, swa::g_status, sizeof word) != cudaSuccess ||
        cudaMemcpyToSymbol(swa::g_status, &zero, sizeof zero) != cudaSuccess) {
        cudaGetLastError();
        return SWA_ERR_CUDA;
    }
    if (detail) *detail = word;
    if (word == 0) return SWA_OK;
    return (word & 0xffu) == swa::kErrTimeout ? SWA_ERR_TIMEOUT : SWA_ERR_CUDA;
}

}  // extern "C"

// ------------------------------------------------------ entry point that allocates nothing
//
// Scratch for swa_attn_fwd_noalloc(): a fixed device array in this module.  Every GPU that
// loads the library holds these bytes until the process exits.  Host code must not use the
// array's name as a device address; the address comes from cudaGetSymbolAddress() below.

namespace {

constexpr size_t kStaticScratchBytes = 64ull << 20;   // 64 MiB
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
void* g_static_ptr[64] = {nullptr};

// Once per device, with that device current: the device address of the scratch array.
int static_scratch(int dev, uint8_t** out) {
    if (dev < 0 || dev >= 64) return SWA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return SWA_ERR_CUDA;
        }
        g_static_ptr[dev] = p;
    }
    *out = static_cast<uint8_t*>(g_static_ptr[dev]);
    return SWA_OK;
}

}  // namespace

extern "C" size_t swa_attn_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

extern "C" int swa_attn_fwd_noalloc(const void* q, const void* k, const void* v, const void* ve,
                                    const void* gate_x, const void* Wg, void* out, float* lse,
                                    int B, int T, int H, int D, int window, float rope_base,
                                    float eps, swa_stream_t stream) {
    Shape s;
    int rc = check_sizes(B, T, H, D, &s);
    if (rc == SWA_OK) rc = check_layer_args(q, k, v, ve, gate_x, Wg, rope_base, eps);
    if (rc == SWA_OK) rc = check_outputs(out, lse);
    if (rc != SWA_OK) return rc;
    const bool has_ve = ve != nullptr;
    const WsLayout L = ws_layout(s, has_ve);
    if (L.total > kStaticScratchBytes) return SWA_ERR_NO_MEMORY;   // beyond the fixed scratch
    int dev;
    if ((rc = device_ready(&dev)) != SWA_OK) return rc;
    uint8_t* ws = nullptr;
    if ((rc = static_scratch(dev, &ws)) != SWA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Every section of the scratch this call reads is written earlier in the same call (the RoPE
    // tables, then khat / v' and the gate; the prologue also zeroes the attention kernel's
    // scheduler counters), so nothing left by an earlier call is read.
    if ((rc = launch_rope_table(ws, L, s, rope_base, st)) != SWA_OK) return rc;
    if ((rc = launch_prologue(q, k, v, ve, gate_x, Wg, ws, L, s, eps, st)) != SWA_OK) return rc;
    return launch_attention(dev, v, has_ve, out, lse, s, window, ws, L, st);
}
