/*
 * lazyflash.h -- C ABI of the LazyFlash attention hot path on B200 (sm_100a).
 *
 * LazyFlash ("LazyFlash allège la rétropropagation de l'attention, 5,72 fois",
 * gyom.fr, 26 Oct 2026) keeps the attention forward exactly dense and makes
 * only the backward block-sparse: query blocks are ranked by the norm of their
 * output gradient, a budget delta bounds the share of gradient mass that may be
 * discarded, each block is kept with probability proportional to its gradient,
 * kept blocks are reweighted so the gradient stays unbiased, and dropped tiles
 * are never loaded or computed.
 *
 * Three calls make up one training step of one attention layer:
 *   lf_attn_fwd      dense forward: O and the per-row log-sum-exp;
 *   lf_block_select  block norms ||dO_b||, D = rowsum(dO * O), the budgeted
 *                    threshold tau, the random keep mask, the 1/p weights and
 *                    the compacted kept-block lists;
 *   lf_attn_bwd      the backward over kept query blocks only.
 *
 * Conventions shared by every call
 *   Layout ("THD"): every token tensor is [T][H][d] row-major and contiguous,
 *     bf16 (q, o, dout, dq: H = hq; k, v, dk, dv: H = hkv).  Segments (packed
 *     variable-length sequences) are delimited by cu_seqlens: int32, nseq + 1
 *     entries, cu_seqlens[0] = 0, non-decreasing, cu_seqlens[nseq] =
 *     total_tokens.  Attention never crosses a segment; with causal != 0 key u
 *     is visible to query t iff u <= t within the segment.
 *   Query head h reads KV head h / (hq / hkv) (consecutive groups, GQA).
 *   lse and D are fp32 [hq][T].  Per-block arrays are [nseq][hq][nbmax] with
 *     nbmax = ceil(max_seqlen / block_q); block i of segment s covers rows
 *     cu_seqlens[s] + i*block_q ... (the last block of a segment may be short);
 *     entries past a segment's block count are written as 0 (kept_idx: -1).
 *   Pointers: all tensor pointers are DEVICE pointers owned by the caller, and
 *     must be 16-byte aligned.  The library allocates no memory and keeps no
 *     per-call state; scratch memory is the caller's workspace (ws, ws_bytes),
 *     sized by lf_workspace_size.
 *   Ordering: every call only enqueues work on `stream` and returns.
 *   Errors: argument errors are returned synchronously, before anything is
 *     launched (LF_ERR_INVALID_ARG, LF_ERR_UNSUPPORTED, LF_ERR_WORKSPACE).
 *     A failed launch returns LF_ERR_CUDA.  Kernels never hang: a kernel whose
 *     bounded wait expired (LF_ERR_TIMEOUT), or that found cu_seqlens
 *     inconsistent with total_tokens / max_seqlen (LF_ERR_INVALID_ARG), records
 *     the failure in a device flag and returns.  The failure is reported
 *     (1) by the next call of any entry point made after the failing call's
 *     work finished: every call that launches work ends with a one-thread
 *     kernel that copies the flag into a page of host memory mapped into the
 *     device, so this check needs no synchronization; that call returns the
 *     code and launches nothing; every later call does the same until the
 *     failure is cleared; and (2) by lf_sync_status (alias
 *     lf_check_device_error), which synchronizes the stream, returns the code
 *     and clears it.  The flag is one per process, shared by all streams and
 *     devices: it reports a failure of any earlier call, not only of the
 *     caller's stream.
 *   Set-up: the first call that launches work on a device maps the host page
 *     (once per process) and stores its device address on that device (a
 *     synchronous copy); make that first call before any stream capture.
 *   Thread safety: calls are reentrant; concurrent calls on different streams
 *     must use different workspaces and outputs.
 */
#ifndef LAZYFLASH_H
#define LAZYFLASH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* lf_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    LF_OK = 0,
    LF_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent sizes, delta outside [0,1) */
    LF_ERR_UNSUPPORTED = 2,  /* a shape this build does not implement (d, block_q) */
    LF_ERR_WORKSPACE = 3,    /* ws_bytes below lf_workspace_size() */
    LF_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
    LF_ERR_TIMEOUT = 5       /* a device-side bounded wait expired (see lf_check_device_error) */
} lf_status;

typedef struct {
    int32_t nseq;               /* number of packed segments, >= 1 */
    const int32_t* cu_seqlens;  /* DEVICE pointer, nseq + 1 int32 offsets */
    int32_t max_seqlen;         /* >= the longest segment (host value) */
    int32_t total_tokens;       /* T = cu_seqlens[nseq] (host value), >= 0 */
    int32_t hq, hkv, d;         /* query heads, KV heads (hq % hkv == 0), head dim (64 or 128) */
    float softmax_scale;        /* scores are softmax_scale * <q, k>; usually 1/sqrt(d) */
    int32_t causal;             /* 1: causal within each segment; 0: full within each segment */
    int32_t block_q;            /* query rows per selection block: 64 or 128 */
} lf_attn_desc;

enum { LF_WS_FWD = 0, LF_WS_SELECT = 1, LF_WS_BWD = 2 };

/* Flags of lf_block_select. */
#define LF_SELECT_NORMS_GIVEN 0x1u  /* block_norm is an input; the norm pass only computes D */

/* Bytes of workspace the call `which` (LF_WS_*) needs for `desc`.
 * Returns LF_ERR_INVALID_ARG / LF_ERR_UNSUPPORTED for a bad descriptor. */
lf_status lf_workspace_size(const lf_attn_desc* desc, int which, size_t* bytes);

/* Dense attention forward (the LazyFlash forward is FlashAttention's,
 * unchanged: article standfirst and section "Le passage arrière fait deux fois
 * le travail du passage avant").
 *   q [T][hq][d], k, v [T][hkv][d] bf16 in; o [T][hq][d] bf16 out;
 *   lse [hq][T] fp32 out: natural-log log-sum-exp of softmax_scale * <q_t, k_u>
 *   over the keys row t sees.
 *   Rows of o/lse outside every segment are left untouched. */
lf_status lf_attn_fwd(const lf_attn_desc* desc, const void* q, const void* k, const void* v,
                      void* o, float* lse, void* ws, size_t ws_bytes, lf_stream_t stream);

/* LazyFlash selection (article section "Un budget sur la masse de gradient, et
 * un tirage qui garde le gradient non biaisé"), per (segment s, head h):
 *   block_norm[s][h][i] = ||dO rows of block i||_F (fp32 accumulation; an input
 *     when flags has LF_SELECT_NORMS_GIVEN);
 *   D[h][t] = sum_c dO[t][h][c] * O[t][h][c] (fp32, unweighted);
 *   tau[s][h] (fp64) = the largest threshold whose expected discarded mass
 *     sum_i (1 - min(1, m_i/tau)) m_i is <= delta * sum_i m_i, found by 64
 *     bisection steps on [0, max_i m_i / (1 - delta)]; each step tests the
 *     inequality multiplied through by the midpoint t, sum_i [m_i < t]
 *     (m_i t - m_i^2) <= (delta M) t, in fp64 with one fused multiply-add per
 *     block and a fixed summation order, so that the result is reproducible
 *     bit for bit; 0 when delta == 0 or all norms are 0 (keep all);
 *   p_i = min(1, m_i / tau) (1 when tau == 0); keep_i = 1 iff p_i >= 1 or
 *     u24 < p_i * 2^24, u24 = word 0 of Philox4x32-10(counter = (i, h, s,
 *     step mod 2^32), key = (seed lo 32, seed hi 32)) >> 8;
 *   block_weight[s][h][i] = (float)(1 / p_i) if kept else 0;
 *   keep (uint8), kept_idx (int32, ascending kept block indices, -1 padded),
 *   kept_cnt[s][h] (int32).
 *   delta must lie in [0, 1).  dout and o are [T][hq][d] bf16.  D may be NULL: the
 *   norm pass then reads dout only (o may be NULL as well), and lf_attn_bwd, given
 *   D = NULL, computes D itself for the rows of kept blocks.  With
 *   LF_SELECT_NORMS_GIVEN and D = NULL no norm pass runs (dout may be NULL). */
lf_status lf_block_select(const lf_attn_desc* desc, const void* dout, const void* o,
                          double delta, uint64_t seed, uint64_t step, uint32_t flags,
                          float* block_norm, float* D, double* tau, float* block_weight,
                          uint8_t* keep, int32_t* kept_idx, int32_t* kept_cnt,
                          void* ws, size_t ws_bytes, lf_stream_t stream);

/* Selection rules of lf_block_select_rule. */
enum {
    LF_RULE_BUDGET = 0,          /* the LazyFlash rule of lf_block_select; param = delta in [0, 1) */
    LF_RULE_FIXED_FRACTION = 1,  /* param = f in (0, 1]: tau = the largest threshold whose expected
                                    kept count sum_i min(1, m_i/tau) reaches f * n (64 bisection
                                    steps, each testing sum_i min(t, m_i) >= (f n) t in the same
                                    fixed order); same Philox draw and 1/p weights as the budget
                                    rule; tau = 0 (keep all) when f = 1 */
    LF_RULE_TOPK = 2             /* param = f in (0, 1]: keep the k = ceil(f * n) largest norms
                                    (ties to the lower index) with weight 1, no draw; tau = the
                                    k-th largest norm */
};

/* Block selection by one of the rules the article compares at equal backward
 * time, "in the same CUDA implementation" (section "Le choix des blocs pèse
 * plus que la quantité sautée"): the adaptive budget, a fraction fixed for the
 * whole run, and top-k.  Outputs, layouts and errors are those of
 * lf_block_select (which is rule LF_RULE_BUDGET); the backward consumes them
 * unchanged.  LF_ERR_INVALID_ARG for an unknown rule or param out of range. */
lf_status lf_block_select_rule(const lf_attn_desc* desc, const void* dout, const void* o,
                               int rule, double param, uint64_t seed, uint64_t step,
                               uint32_t flags, float* block_norm, float* D, double* tau,
                               float* block_weight, uint8_t* keep, int32_t* kept_idx,
                               int32_t* kept_cnt, void* ws, size_t ws_bytes, lf_stream_t stream);

/* LazyFlash backward over kept query blocks (article sections "Le passage
 * arrière ..." and "Un budget sur la masse de gradient ...": dropped tiles are
 * never loaded or computed; kept blocks' output gradient is scaled by
 * block_weight).  With dO~ = w_b(t) dO_t and P the softmax of the forward:
 *   dP = dO~ V^T, dS = P * (dP - w D), dQ = scale dS K, dK = scale dS^T Q
 *   (summed over the hq/hkv query heads of a KV head), dV = P^T dO~.
 *   q, k, v, dout bf16 in (layouts as above); lse, D fp32 [hq][T] from
 *   lf_attn_fwd / lf_block_select (D may be NULL: it is then computed from o
 *   and dout into the workspace, for the rows of kept blocks only, the others
 *   being 0; o may be NULL when D is given);
 *   block_weight, kept_idx, kept_cnt from lf_block_select;
 *   dq [T][hq][d], dk, dv [T][hkv][d] bf16 out.  Rows of dropped blocks get
 *   dq = 0; dk/dv rows no kept block reaches get 0.  The rows of q and dout that
 *   belong to dropped blocks are never read (at 64-row granularity when
 *   block_q = 64), except rows that fall inside the last tile of the previous
 *   segment (a segment's last 128-row tile, or 64-row half, also loads the rows
 *   after the segment's end; they are masked with P = 0).  Inputs must be finite:
 *   a non-finite value in those rows, or in the k/v rows after a segment's end
 *   within its last tile, can turn the masked products into NaN. */
lf_status lf_attn_bwd(const lf_attn_desc* desc, const void* q, const void* k, const void* v,
                      const void* o, const float* lse, const void* dout, const float* D,
                      const float* block_weight, const int32_t* kept_idx,
                      const int32_t* kept_cnt, void* dq, void* dk, void* dv,
                      void* ws, size_t ws_bytes, lf_stream_t stream);

/* Capacity of the library's static scratch array used by lf_attn_bwd_static_ws. */
#define LF_STATIC_WS_BYTES ((size_t)32 << 20)

/* lf_attn_bwd without a workspace argument and without any allocation.
 * The paper has no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory on the library's behalf: custom-op plugin
 * interfaces that hand an operator only its inputs and outputs, and runtimes
 * that plan all device memory ahead of time or forbid cudaMalloc/cudaFree while
 * they run (those calls synchronize the device and are not allowed inside a
 * stream capture).
 *   Arguments and results are those of lf_attn_bwd.  The scratch (the fp32
 *   accumulators of dQ, dK and dV, plus D when D is NULL) lives in one
 *   file-scope device array of LF_STATIC_WS_BYTES bytes that every GPU loading
 *   the library holds until the process exits.  A problem whose scratch
 *   exceeds it, i.e. 4 * total_tokens * (hq + 2 * hkv) * d bytes (each of the
 *   three parts rounded up to 256), plus 4 * total_tokens * hq when D is NULL,
 *   returns LF_ERR_WORKSPACE before anything is launched.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and keeps it for the life
 *   of the process; make that first call before any stream capture.  A device
 *   reset (cudaDeviceReset, or a framework that destroys and recreates the
 *   primary context) reloads the library's device code, possibly at another
 *   address: do not call this entry point on a device after resetting it.  The call never calls cudaMalloc, cudaFree or an
 *   allocating library routine; the accumulators a call uses are cleared at
 *   its start (dK and dV need none when the query heads of each KV head fit
 *   in one CTA, i.e. hq/hkv is 1, 2 or 4: they are then written directly).
 *   All calls on a device share the one array and it keeps the last call's
 *   contents: calls that may overlap on the GPU (different streams, or host
 *   threads without ordering) race on it and produce wrong dQ. */
lf_status lf_attn_bwd_static_ws(const lf_attn_desc* desc, const void* q, const void* k,
                                const void* v, const void* o, const float* lse, const void* dout,
                                const float* D, const float* block_weight,
                                const int32_t* kept_idx, const int32_t* kept_cnt, void* dq,
                                void* dk, void* dv, lf_stream_t stream);

/* Failure-detection self-test (no counterpart in the article): launches one
 * CTA whose bounded barrier wait, the one every kernel uses, waits for a phase
 * that nothing completes and gives up after 2^limit_log2 SM cycles (10..31),
 * recording a timeout in the device flag.  Nothing faults or traps: after
 * lf_check_device_error returns LF_ERR_TIMEOUT the context stays usable.
 * Returns LF_ERR_INVALID_ARG for a limit outside 10..31. */
lf_status lf_watchdog_selftest(uint32_t limit_log2, lf_stream_t stream);

/* Waits for `stream`, then reads and clears the device-side failure flag (see
 * "Errors" above).  Returns LF_ERR_TIMEOUT if a kernel gave up a bounded wait
 * since the flag was last cleared, LF_ERR_INVALID_ARG if a kernel found
 * cu_seqlens inconsistent with total_tokens / max_seqlen (the first failure is
 * the one reported), LF_ERR_CUDA if the stream reported a CUDA error, else
 * LF_OK.  The flag is shared by all streams and devices of the process, so a
 * check on one stream also reports, and clears, a failure raised by a kernel on
 * another stream. */
lf_status lf_sync_status(lf_stream_t stream);

/* The same function as lf_sync_status (its earlier name). */
lf_status lf_check_device_error(lf_stream_t stream);

/* Static, human-readable name of a status code. */
const char* lf_status_string(lf_status status);

#ifdef __cplusplus
}
#endif

#endif /* LAZYFLASH_H */
