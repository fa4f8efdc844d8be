/*
 * swa_attn.h -- C ABI of the B200 (sm_100a) causal sliding-window attention forward.
 *
 * The layer (one call = one attention layer of the nanochat / modded-NanoGPT speedrun model):
 *
 *   qhat = rms(rope(q)),  khat = rms(rope(k))
 *        intelliparadigm "GPT-2 for $73", section 2.2 (q, k = norm(rope(q)), norm(rope(k)));
 *        section 2.1 (parameter-free RMSNorm); kongchang speedrun explainer, "RoPE" paragraph.
 *        rope: pairs (i, i + D/2), theta_i = rope_base^(-2i/D), position t = 0..T-1 rotates
 *        (a, b) -> (a cos(t theta_i) - b sin(t theta_i), a sin(t theta_i) + b cos(t theta_i)).
 *        rms:  x / sqrt(mean_D(x^2) + eps), no learned scale.
 *   v'   = v + 2 sigmoid(gate_x[b,t,:] . Wg[:, h]) * ve        (value-embedding layers only)
 *        PaperWeekly repost of the nanochat write-up, "Value Embeddings" paragraph.
 *   out  = softmax(qhat khat^T / sqrt(D) + mask) v'
 *        "Let's reproduce GPT-2 (124M)" notes, section 3 (scores, lower-triangular mask that
 *        includes the diagonal, softmax over keys, weighted sum of values).
 *        mask: key j is visible to query i iff 0 <= i - j < W, W = window (intelliparadigm
 *        section 3.2: local windows of 1024 tokens, a full window of 2048 every fourth layer);
 *        window <= 0 or window >= T means full causal.
 *   lse  = ln sum_j exp(qhat_i . khat_j / sqrt(D)) over the visible keys (natural log).
 *
 * Layouts (all row-major, contiguous, no strides):
 *   q, k, v, ve, out : bf16 (B, T, H, D)        -- the native layout (intelliparadigm 3.1)
 *   gate_x           : bf16 (B, T, 32)          -- x[..., :32].contiguous()
 *   Wg               : bf16 [32, H]             -- one gate per head, no bias
 *   lse              : fp32 (B, H, T)
 *
 * Ownership: every pointer is a DEVICE pointer owned by the caller, except where stated.
 * The library never frees a caller pointer and never writes q, k, v, ve, gate_x or Wg.
 *
 * Streams: calls are asynchronous on `stream` (NULL = the legacy default stream) and never
 * synchronise the host, except swa_attn_last_device_status().
 *
 * Threads: calls may come from several host threads at once.  The per-device setup of the first
 * call, the library-owned workspace and the backward's side stream are guarded by locks, and a
 * call that reuses the library workspace on another stream first waits, on the device, for the
 * previous call that used it.  Caller-owned workspaces are the caller's to keep apart.
 *
 * Precision: every qhat, khat and v' element the prologue writes is the correctly rounded bf16
 * (nearest, ties to even) of its exact value, so the tensor-core operands do not depend on how the
 * arithmetic is organised.
 *
 * Errors: a negative swa_status.  Arguments are validated before anything is enqueued; a
 * rejected call has no effect.  Waits inside the kernels are bounded: if one expires, the
 * kernel records SWA_ERR_TIMEOUT in a per-device status word and exits cleanly; read it with
 * swa_attn_last_device_status().
 */
#ifndef SWA_ATTN_H_
#define SWA_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SWA_API __attribute__((visibility("default")))
#else
#define SWA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* swa_stream_t;

typedef enum swa_status {
    SWA_OK = 0,
    SWA_ERR_INVALID_ARG = -1,  /* null pointer, size < 1, bad eps / rope_base, ve/gate_x/Wg partly set */
    SWA_ERR_UNSUPPORTED = -2,  /* D not in {64, 128}, sizes beyond int32 indexing, device not sm_100 */
    SWA_ERR_MISALIGNED = -3,   /* a tensor pointer or the workspace is not 16-byte aligned */
    SWA_ERR_CUDA = -4,         /* a CUDA runtime / driver call failed (launch, allocation by CUDA),
                                  or a kernel found its shared memory misaligned and did nothing */
    SWA_ERR_TIMEOUT = -5,      /* a bounded wait inside a kernel expired (read via last_device_status) */
    SWA_ERR_NO_MEMORY = -6,    /* workspace too small (swa_attn_fwd_ws) or allocation failed */
    SWA_ERR_NO_DEVICE = -7     /* no CUDA device is visible */
} swa_status;

/*
 * Full layer forward.  Steps: RoPE + RMS norm of q and k, gate + add of the value embedding,
 * windowed causal attention, bf16 out and fp32 lse.
 *
 * q, k, v      bf16 (B,T,H,D), read only.
 * ve, gate_x, Wg  value-embedding inputs; all three NULL for a layer without value embeddings,
 *              otherwise all three set (else SWA_ERR_INVALID_ARG).
 * out          bf16 (B,T,H,D), written.
 * lse          fp32 (B,H,T), written; NULL skips it.
 * B, T, H      >= 1;  D in {64, 128};  B*T*H*D < 2^31;  B, H <= 65535 (else SWA_ERR_UNSUPPORTED).
 * window       keys visible to a query, counting itself; <= 0 or >= T is full causal.
 * rope_base    > 0 and finite (10000 in the pages' models).
 * eps          >= 0 and finite (1e-6 here).  At eps = 0 an all-zero q or k head row has no
 *              normalised value (0/0 in the definition): such inputs are outside the domain and
 *              their results are unspecified.
 * stream       CUDA stream (NULL = legacy default stream).
 *
 * Scratch: the library keeps one workspace per device (qhat, khat, v', the gates, the RoPE table),
 * grown on demand with stream-ordered allocation on `stream` and kept until the library is
 * unloaded.  Each call records an event after its kernels; a call on another stream first makes
 * its stream wait for that event, so calls on different streams that share the workspace run one
 * after the other on the GPU (callers that want them to overlap use swa_attn_fwd_ws() with
 * separate workspaces).  Launches: the gate kernel (value-embedding layers), the prologue kernel
 * and the attention kernel, plus the RoPE table when T, D or rope_base changes.
 */
SWA_API int swa_attn_fwd(const void* q, const void* k, const void* v,
                 const void* ve, const void* gate_x, const void* Wg,
                 void* out, float* lse,
                 int B, int T, int H, int D, int window,
                 float rope_base, float eps, swa_stream_t stream);

/*
 * Grouped-query attention (the pages size the key/value projection separately, as kv_dim:
 * intelliparadigm "GPT-2 for $73", model section): as swa_attn_fwd, with q (B,T,H,D) and k, v, ve
 * (B,T,Hkv,D), gate_x
 * (B,T,32), Wg [32,Hkv]; Hkv divides H and query head h attends with key/value head h / (H/Hkv).
 * The prologue runs on the Hkv key/value heads once (not per query head).  Hkv == H is exactly
 * swa_attn_fwd.  Errors as swa_attn_fwd; SWA_ERR_INVALID_ARG if Hkv does not divide H.
 */
SWA_API int swa_attn_fwd_gqa(const void* q, const void* k, const void* v,
                             const void* ve, const void* gate_x, const void* Wg,
                             void* out, float* lse,
                             int B, int T, int H, int Hkv, int D, int window,
                             float rope_base, float eps, swa_stream_t stream);

/*
 * Document-boundary mask (packed documents; the pages list variable-length attention among the
 * changes that were tried: intelliparadigm "GPT-2 for $73", section 7).  As swa_attn_fwd_gqa, plus
 * doc: int32 (B, T) device array of document ids.  A document is a maximal run of equal ids along
 * a sequence (number packed documents in order: ids that never repeat across runs); key j is
 * visible to query i iff 0 <= i - j < window and j is in i's document.  RoPE positions stay the
 * sequence positions 0..T-1.  Key tiles before the first query row's document start are skipped.
 * Uses the library-owned workspace (plus B*T int32 document starts), with its stream ordering.
 * Errors as swa_attn_fwd_gqa; SWA_ERR_INVALID_ARG if doc is NULL, SWA_ERR_MISALIGNED if it is
 * not 4-byte aligned.
 */
SWA_API int swa_attn_fwd_doc(const void* q, const void* k, const void* v,
                             const void* ve, const void* gate_x, const void* Wg, const int* doc,
                             void* out, float* lse,
                             int B, int T, int H, int Hkv, int D, int window,
                             float rope_base, float eps, swa_stream_t stream);

/* Bytes of caller workspace swa_attn_fwd_ws() needs for these sizes (0 on invalid sizes). */
SWA_API size_t swa_attn_workspace_bytes(int B, int T, int H, int D, int has_ve);

/*
 * Byte offset of one section of the workspace, for callers that read the prologue's results
 * (e.g. to keep them for a backward pass) after swa_attn_prologue():
 *   SWA_WS_QHAT, SWA_WS_KHAT   bf16 (B,T,H,D): rms(rope(q)), rms(rope(k)), each element the
 *                              correctly rounded bf16 (nearest, ties to even) of its exact value;
 *   SWA_WS_VPRIME              bf16 (B,T,H,D): v + 2 sigmoid(gate_x . Wg) ve, same rounding
 *                              (value-embedding layers only);
 *   SWA_WS_ROPE_TABLE          the RoPE table (internal format).
 * Returns (size_t)-1 for invalid sizes or a section that does not exist.
 */
enum swa_ws_section { SWA_WS_QHAT = 0, SWA_WS_KHAT = 1, SWA_WS_VPRIME = 2, SWA_WS_ROPE_TABLE = 3 };
SWA_API size_t swa_attn_workspace_offset(int B, int T, int H, int D, int has_ve, int section);

/*
 * Same as swa_attn_fwd() with caller-owned device scratch: `workspace` (16-byte aligned,
 * at least swa_attn_workspace_bytes() bytes) holds qhat, khat, v', the gates and the RoPE table, which
 * is rebuilt on every call (one small extra kernel).  It runs swa_attn_rope_table(),
 * swa_attn_prologue() and swa_attn_attention().  Nothing is allocated.
 * SWA_ERR_NO_MEMORY if ws_bytes is too small.
 */
SWA_API int swa_attn_fwd_ws(const void* q, const void* k, const void* v,
                    const void* ve, const void* gate_x, const void* Wg,
                    void* out, float* lse,
                    int B, int T, int H, int D, int window,
                    float rope_base, float eps,
                    void* workspace, size_t ws_bytes, swa_stream_t stream);

/*
 * The steps of swa_attn_fwd_ws(), exposed for per-stage timing and tests.
 *
 * swa_attn_rope_table: fill the workspace's RoPE table, cos/sin(t * rope_base^(-2i/D)) for
 *   t < T, i < D/2, evaluated in fp64 and stored as fp32.  It depends only on T, D and
 *   rope_base, so a caller that keeps one workspace for many calls of the same T, D and base
 *   builds it once (swa_attn_fwd does that with its own workspace).
 * swa_attn_prologue: RoPE + RMS norm of q and k, gate + add of the value embedding, into the
 *   workspace (same sizes and rules as swa_attn_fwd_ws).  Uses the table already in the
 *   workspace; it does not rebuild it.  It also resets the scheduler counters the attention kernel
 *   takes its work from.
 * swa_attn_attention: the windowed attention on a workspace that swa_attn_prologue() filled
 *   for the same B, T, H, D and value-embedding setting (`v` is read directly when has_ve == 0).
 * All of them: asynchronous on `stream`, validation before any launch, errors as swa_attn_fwd_ws.
 */
SWA_API int swa_attn_rope_table(int B, int T, int H, int D, int has_ve, float rope_base,
                                void* workspace, size_t ws_bytes, swa_stream_t stream);

SWA_API int swa_attn_prologue(const void* q, const void* k, const void* v,
                      const void* ve, const void* gate_x, const void* Wg,
                      int B, int T, int H, int D, float rope_base, float eps,
                      void* workspace, size_t ws_bytes, swa_stream_t stream);

SWA_API int swa_attn_attention(const void* v, int has_ve, void* out, float* lse,
                       int B, int T, int H, int D, int window,
                       void* workspace, size_t ws_bytes, swa_stream_t stream);


/*
 * swa_attn_fwd_noalloc: swa_attn_fwd() for callers that cannot allocate device memory on the
 * call path -- a plugin whose host framework owns all device memory and forbids allocation
 * inside its execute call, or a latency-critical loop where an allocation (which may
 * synchronise the device) is not allowed.  The pages have no counterpart of this entry point.
 *
 * The caller passes inputs and outputs exactly as for swa_attn_fwd(), and the call computes the
 * same result with the same kernels; the scratch (qhat, khat, v', the gates and the RoPE table) lives in
 * a fixed device array compiled into the library, swa_attn_noalloc_scratch_bytes() bytes (64 MiB).
 * Nothing is allocated or freed by the call itself.
 *   - CUDA loads the library's device code, and with it the array, on a device when the library
 *     is first used there (lazy module loading): from then on that device holds the 64 MiB until
 *     the process exits, and that first use may itself allocate.  The first call of
 *     swa_attn_fwd_noalloc() on a device also looks up the array's device address (a runtime query,
 *     once per device, with that device current).  Callers that must not allocate make one warm-up
 *     call on each device outside their no-allocation region and before any stream capture.
 *   - Sizes whose workspace (swa_attn_workspace_bytes()) exceeds that array are rejected with
 *     SWA_ERR_NO_MEMORY before anything is enqueued.
 *   - All calls on a device share the one array and it keeps the last call's contents; every
 *     byte a call reads is written earlier in that call.  Calls that overlap on the GPU (other
 *     streams, other host threads) race on it: serialise them.
 */
SWA_API int swa_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                 const void* ve, const void* gate_x, const void* Wg,
                                 void* out, float* lse,
                                 int B, int T, int H, int D, int window,
                                 float rope_base, float eps, swa_stream_t stream);

/* Size in bytes of the fixed scratch array behind swa_attn_fwd_noalloc(). */
SWA_API size_t swa_attn_noalloc_scratch_bytes(void);

/* Static description of a status code (never NULL). */
SWA_API const char* swa_attn_strerror(int status);

/*
 * Synchronises `stream`, then returns and clears the current device's status word:
 * SWA_OK, SWA_ERR_TIMEOUT (a bounded wait expired in some kernel since the last read) or
 * SWA_ERR_CUDA (the stream reported an error).  If `detail` is not NULL it receives the raw
 * word (bits 0-7 kind, 8-15 wait site, 16-31 block index).
 */
SWA_API int swa_attn_last_device_status(swa_stream_t stream, unsigned int* detail);

/*
 * One generation step with a key/value cache (the pages list a KV cache among the missing
 * pieces: "Let's reproduce GPT-2 (124M)" notes, section 19).  For the new token of every
 * sequence, at position `pos` (the same for all b):
 *   1. the prologue of swa_attn_fwd at position pos: qhat = RMS(RoPE(q, pos)),
 *      khat = RMS(RoPE(k, pos)), v' = v + 2 sigmoid(gate_x . Wg[:, h]) ve (value-embedding
 *      layers) or v; khat and v' are written to k_cache[b, pos, h, :] and v_cache[b, pos, h, :],
 *      bit-identical to what the prefill path computes for that token;
 *   2. attention of qhat over the cached keys j in [max(0, pos - W + 1), pos] (W = Tmax if
 *      window <= 0 or window >= Tmax): out[b,h,:] = sum_j softmax_j(qhat . khat_j / sqrt(D)) v'_j,
 *      lse[b,h] = ln sum_j exp(qhat . khat_j / sqrt(D)).
 * Arguments:
 *   q, k, v      bf16 (B, H, D): the new token's raw projections.
 *   ve, gate_x, Wg  bf16 (B, H, D) / (B, 32) / (32, H), all set (value-embedding layer) or all NULL.
 *   k_cache, v_cache  bf16 (B, Tmax, H, D), caller-owned: entries j < pos (inside the window) must
 *                hold khat / v' of earlier positions (as written by earlier calls or by the prefill
 *                path); entry pos is written.
 *   out          bf16 (B, H, D), written.   lse  fp32 (B, H) or NULL.
 *   workspace    device memory of at least swa_attn_decode_workspace_bytes(B, Tmax, H, D, has_ve,
 *                window) bytes, 16-byte aligned, caller-owned and not retained.
 * Scores, exponentials and weighted sums are fp32 (no bf16 rounding of the weights).  The call is
 * asynchronous on `stream` (two kernels: the token's key/value prologue, then one cluster of CTAs
 * per row for the attention, which also forms qhat); arguments are validated before anything is
 * enqueued.  Errors: SWA_ERR_INVALID_ARG (null pointer, pos outside [0, Tmax), bad rope_base /
 * eps, partial value-embedding set), SWA_ERR_UNSUPPORTED (D not 64/128, sizes beyond int32),
 * SWA_ERR_MISALIGNED, SWA_ERR_NO_MEMORY (workspace too small), SWA_ERR_CUDA.
 */
SWA_API size_t swa_attn_decode_workspace_bytes(int B, int Tmax, int H, int D, int has_ve, int window);
SWA_API int swa_attn_decode(const void* q, const void* k, const void* v, const void* ve,
                            const void* gate_x, const void* Wg, void* k_cache, void* v_cache,
                            int pos, void* out, float* lse, int B, int Tmax, int H, int D,
                            int window, float rope_base, float eps, void* workspace,
                            size_t ws_bytes, swa_stream_t stream);
/* Grouped-query decode step: as swa_attn_decode with q (B, H, D) and k, v, ve (B, Hkv, D),
 * gate_x (B, 32), Wg (32, Hkv), caches (B, Tmax, Hkv, D); Hkv divides H and query head h attends
 * with key/value head h / (H / Hkv).  The workspace size is that of swa_attn_decode for (B, Tmax,
 * H, D).  SWA_ERR_INVALID_ARG if Hkv does not divide H. */
SWA_API int swa_attn_decode_gqa(const void* q, const void* k, const void* v, const void* ve,
                                const void* gate_x, const void* Wg, void* k_cache, void* v_cache,
                                int pos, void* out, float* lse, int B, int Tmax, int H, int Hkv,
                                int D, int window, float rope_base, float eps, void* workspace,
                                size_t ws_bytes, swa_stream_t stream);

/*
 * One generation step of the document-masked layer: as swa_attn_decode_gqa, plus doc_start, an
 * int32 (B,) device array with the first position of each sequence's current document (the
 * document the new token at `pos` belongs to; values above pos are read as pos).  The new token
 * attends to the cached keys [max(pos - W + 1, doc_start[b]), pos] (the document-boundary mask of
 * swa_attn_fwd_doc, row pos).  doc_start = NULL is swa_attn_decode_gqa.  SWA_ERR_MISALIGNED if
 * doc_start is not 4-byte aligned.
 */
SWA_API int swa_attn_decode_doc(const void* q, const void* k, const void* v,
                                const void* ve, const void* gate_x, const void* Wg,
                                void* k_cache, void* v_cache, int pos, const int* doc_start,
                                void* out, float* lse,
                                int B, int Tmax, int H, int Hkv, int D, int window,
                                float rope_base, float eps,
                                void* workspace, size_t ws_bytes, swa_stream_t stream);

/*
 * The layer from its input x: the bias-free q, k, v projection fused with the prologue, then the
 * attention of swa_attn_fwd_gqa.  The pages form q, k, v of each layer as linear maps of the
 * layer input ("Let's reproduce GPT-2 (124M)" notes, section 3, the attention listing;
 * intelliparadigm "GPT-2 for $73", section 2: separate bias-free maps, key/value width kv_dim):
 *   y = x Wqkv^T (fp32 tensor-core accumulation, never rounded or stored), then
 *   qhat = RMS(RoPE(y_q)), khat = RMS(RoPE(y_k)), v' = y_v + 2 sigmoid(x[..., :32] . Wg[:, h]) ve.
 * Arguments (device pointers, caller-owned):
 *   x        bf16 (B, T, C) contiguous, C a multiple of 8 (at least 32 with the value embedding).
 *   Wqkv     bf16 [(H + 2 Hkv) D, C], the linear layer's layout: rows 0 .. H D - 1 give q (head h at
 *            rows h D ..), then Hkv D rows of k, then Hkv D rows of v.
 *   ve, Wg   bf16 (B, T, Hkv, D) gathered value-embedding rows and [32, Hkv], both set or both NULL.
 * swa_attn_qkv_prologue writes qh bf16 (B, T, H, D), kh and vp bf16 (B, T, Hkv, D) (caller buffers);
 * swa_attn_fwd_x writes out bf16 (B, T, H, D) and lse fp32 (B, H, T) (NULL = skip) with qhat, khat,
 * v' kept in the workspace.  workspace: at least swa_attn_fwd_x_workspace_bytes(B, T, H, Hkv, D)
 * bytes, 16-byte aligned, nothing kept between calls.  Both calls leave the workspace's RoPE table
 * in their own form (fp32 cos and sin, no fp64 copy): on a workspace they used, call
 * swa_attn_rope_table() again before swa_attn_prologue().  Asynchronous on `stream`; arguments are
 * validated before anything is enqueued.  Errors: SWA_ERR_INVALID_ARG (null pointer, ve / Wg not
 * both set, C < 32 with the value embedding, Hkv not dividing H, bad rope_base / eps),
 * SWA_ERR_UNSUPPORTED (D not 64 / 128, C not a multiple of 8, B T H D or B T C at least 2^31),
 * SWA_ERR_MISALIGNED, SWA_ERR_NO_MEMORY, SWA_ERR_CUDA.
 */
SWA_API size_t swa_attn_fwd_x_workspace_bytes(int B, int T, int H, int Hkv, int D);
SWA_API int swa_attn_qkv_prologue(const void* x, const void* Wqkv, const void* ve, const void* Wg,
                                  void* qh, void* kh, void* vp, int B, int T, int C, int H, int Hkv,
                                  int D, float rope_base, float eps, void* workspace, size_t ws_bytes,
                                  swa_stream_t stream);
SWA_API int swa_attn_fwd_x(const void* x, const void* Wqkv, const void* ve, const void* Wg, void* out,
                           float* lse, int B, int T, int C, int H, int Hkv, int D, int window,
                           float rope_base, float eps, void* workspace, size_t ws_bytes,
                           swa_stream_t stream);

/*
 * Backward of the layer: the gradient of loss = sum(dout * out) + sum(dlse * lse) for the layer of
 * swa_attn_fwd / swa_attn_fwd_gqa (the pages train it end to end; the log-sum-exp the forward
 * writes lets the backward rebuild the softmax: "Let's reproduce GPT-2 (124M)" notes, the
 * attention-kernel discussion in section 19).  Per visible pair (i, j) with P_ij = exp(s_ij - lse_i):
 *   dP_ij = dout_i . v'_j,  delta_i = dout_i . out_i,  dS_ij = P_ij (dP_ij - delta_i + dlse_i),
 *   dqhat_i = sum_j dS_ij khat_j / sqrt(D),  dkhat_j = sum_i dS_ij qhat_i / sqrt(D),
 *   dv'_j = sum_i P_ij dout_i  (summed over the query heads of a key/value head's group),
 * then the prologue in reverse: dq = RoPE^T(r dqhat - (r^3/D)(x . dqhat) x) per row (likewise dk),
 * dv = dv', dve = g dv', dz = (dv' . ve) 2 sigmoid(z)(1 - sigmoid(z)), dgate_x = dz Wg^T,
 * dWg = gate_x^T dz.
 * Arguments (device pointers, caller-owned, all read-only except the gradients and workspace):
 *   q, k, v, ve, gate_x, Wg   the forward's inputs, shapes as swa_attn_fwd_gqa.
 *   out, lse                  the forward's outputs for these inputs: bf16 (B,T,H,D), fp32 (B,H,T).
 *   dout                      bf16 (B,T,H,D).   dlse  fp32 (B,H,T), or NULL for zero.
 *   dq                        bf16 (B,T,H,D), written.   dk, dv  bf16 (B,T,Hkv,D), written.
 *   dve                       bf16 (B,T,Hkv,D): gradient of the looked-up value-embedding rows.
 *   dgate_x                   fp32 (B,T,32).   dWg  fp32 (32,Hkv).
 *                             These three are set on value-embedding layers and NULL otherwise.
 *   workspace                 at least swa_attn_bwd_workspace_bytes(B,T,H,Hkv,D,has_ve) bytes,
 *                             16-byte aligned; nothing in it is kept between calls.
 * qhat, khat and v' are recomputed by the forward's prologue (bit-identical to the forward's);
 * P and dS enter the tensor-core products as bf16 (round to nearest), accumulation is fp32.
 * Asynchronous on `stream` (about ten kernels); arguments are validated before anything is
 * enqueued.  Errors: SWA_ERR_INVALID_ARG (null pointer, value-embedding gradients not matching the
 * inputs, Hkv not dividing H, bad rope_base / eps), SWA_ERR_UNSUPPORTED, SWA_ERR_MISALIGNED,
 * SWA_ERR_NO_MEMORY (workspace too small), SWA_ERR_CUDA; bounded-wait timeouts inside the kernels
 * are reported by swa_attn_last_device_status().
 */
SWA_API size_t swa_attn_bwd_workspace_bytes(int B, int T, int H, int Hkv, int D, int has_ve);
SWA_API int swa_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* ve,
                             const void* gate_x, const void* Wg, const void* out, const float* lse,
                             const void* dout, const float* dlse, void* dq, void* dk, void* dv,
                             void* dve, float* dgate_x, float* dWg, int B, int T, int H, int Hkv,
                             int D, int window, float rope_base, float eps, void* workspace,
                             size_t ws_bytes, swa_stream_t stream);

/*
 * The backward of the document-masked layer (swa_attn_fwd_doc): as swa_attn_bwd_gqa, plus doc, the
 * same int32 (B, T) document ids the forward took (documents are maximal runs of equal ids).  The
 * query-tile kernel skips key tiles before the tile's first document start and masks keys before
 * each row's document start; the key-tile kernel skips query tiles past the tile's last document end
 * and masks queries past each key's document end.  Workspace: swa_attn_bwd_workspace_bytes() (it
 * reserves the document starts and ends).  doc = NULL is swa_attn_bwd_gqa.  SWA_ERR_MISALIGNED if
 * doc is not 4-byte aligned.
 */
SWA_API int swa_attn_bwd_doc(const void* q, const void* k, const void* v, const void* ve, const void* gate_x,
                             const void* Wg, const int* doc, const void* out, const float* lse,
                             const void* dout, const float* dlse, void* dq, void* dk, void* dv, void* dve,
                             float* dgate_x, float* dWg, int B, int T, int H, int Hkv, int D, int window,
                             float rope_base, float eps, void* workspace, size_t ws_bytes,
                             swa_stream_t stream);
/*
 * swa_attn_bwd_saved: the multi-head backward (as swa_attn_bwd) for a caller that keeps the
 * forward's activations.  Use it when `workspace` (swa_attn_bwd_workspace_bytes() bytes, which
 * covers swa_attn_workspace_bytes()) was passed to the swa_attn_fwd_ws() call that produced `out`
 * and `lse`, with the same q, k, v, ve, gate_x, Wg, sizes, rope_base and eps, and nothing has
 * written to it since.  That call left qhat, khat, v', the gates and the RoPE tables at the
 * offsets this backward reads, so the prologue is not recomputed.  The gradients are bit-identical
 * to swa_attn_bwd's.  The call cannot check that the workspace holds this layer's forward state:
 * any other content gives wrong gradients (every access stays inside the workspace).
 */
SWA_API int swa_attn_bwd_saved(const void* q, const void* k, const void* v, const void* ve,
                               const void* gate_x, const void* Wg, const void* out, const float* lse,
                               const void* dout, const float* dlse, void* dq, void* dk, void* dv,
                               void* dve, float* dgate_x, float* dWg, int B, int T, int H, int D,
                               int window, float rope_base, float eps, void* workspace, size_t ws_bytes,
                               swa_stream_t stream);

/* The multi-head layer: swa_attn_bwd_gqa with Hkv = H. */
SWA_API int swa_attn_bwd(const void* q, const void* k, const void* v, const void* ve,
                         const void* gate_x, const void* Wg, const void* out, const float* lse,
                         const void* dout, const float* dlse, void* dq, void* dk, void* dv, void* dve,
                         float* dgate_x, float* dWg, int B, int T, int H, int D, int window,
                         float rope_base, float eps, void* workspace, size_t ws_bytes,
                         swa_stream_t stream);

/*
 * Failure-detection self-test (no counterpart in the pages).  Enqueues on `stream` one block of
 * 32 threads that waits, through the bounded wait every kernel here uses, on an mbarrier that
 * nothing ever completes.  After `limit_ms` (1..10000) the wait gives up, records SWA_ERR_TIMEOUT
 * at wait site 30 in the device status word and the kernel returns normally: the device context
 * stays usable.  Read the result with swa_attn_last_device_status().  Returns SWA_OK once the
 * kernel is enqueued, SWA_ERR_INVALID_ARG for a limit out of range, else as the other calls.
 */
SWA_API int swa_attn_selftest_wait(int limit_ms, swa_stream_t stream);

/* Upper bound, in milliseconds, on any single wait inside the kernels (default 2000).
 * Returns the previous value.  Values < 1 are ignored. */
SWA_API int swa_attn_set_wait_limit_ms(int ms);

/* ABI version: major * 10000 + minor * 100 + patch. */
SWA_API int swa_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SWA_ATTN_H_ */
