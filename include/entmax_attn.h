/*
 * entmax_attn.h - C ABI of libentmax_attn.so: alpha-entmax attention on NVIDIA B200 (sm_100a).
 *
 * What the library computes (AdaSplash-2, "Faster Differentiable Sparse Attention"):
 *
 *   s_ij = scale * q_i . k_j,  z_ij = (alpha - 1) s_ij          (j <= i when causal)
 *   p_ij = [z_ij - tau_i]_+^(1/(alpha-1)),  with tau_i such that sum_j p_ij = 1
 *   O_i  = sum_j p_ij v_j
 *
 * alpha-entmax replaces the softmax normaliser and yields exact zeros, at the cost of a root search
 * for tau (gist.science (de) summary, section 1 "Problemstellung"; euno.news summary, "方法论" item 1).
 * The forward builds an on-chip score histogram per query row whose left-edge root tau_h is a lower
 * bound on tau (gist.science (de), section 2, "Streaming & Histogramm-Erstellung", "Theoretische
 * Garantie"), refines it with a safeguarded Halley / Newton / secant solver with bisection fallback
 * ("Hybrid Solver & Sparsity-Awareness"), records the nonzero (query block, key block) pairs in a
 * bit-packed mask, 32 key blocks per uint32 ("Bit-Packed Block Mask"), and computes P V only on those
 * blocks (or, where every row of a 128-row tile was solved on chip and has a small support, as a sum over
 * the support entries gathered from V in fp32). The backward walks the same mask ("GPU-Optimierung":
 * find-next-set and popcount over the nonzero blocks) with the entmax Jacobian dS = u (g - delta),
 * u = p^(2 - alpha) on the support, g = dO V^T, delta = sum(u g) / sum(u).
 *
 * Conventions for every entry point
 *   - Tensors are [B, H, n, d] row-major, d fastest, on the current CUDA device. bf16 tensors use
 *     the IEEE bfloat16 bit layout. Base addresses must be 16-byte aligned (TMA), else
 *     ENTMAX_ERR_ALIGN.
 *   - tau, lse, and per-row statistics are float32 [B, H, n].
 *   - block_mask is uint32 [B, H, nqb, nw] with nqb = ceil(n / mb), nkb = ceil(n / mb),
 *     nw = ceil(nkb / 32); bit (J % 32) of word J / 32 in row I is set when some entry of query
 *     block I and key block J is nonzero. mb is the mask block (opts->mask_block).
 *   - All device buffers are owned by the caller. The library allocates and frees nothing, and does
 *     not synchronise: calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream).
 *   - Argument errors return before any launch, with no effect. A device-side wait that runs out
 *     (a pipeline barrier that does not complete within about two seconds) makes the kernel record
 *     ENTMAX_ERR_TIMEOUT in a device status word and return early; entmax_attn_check() reports it.
 *   - No C++ exception crosses this boundary.
 */
#ifndef ENTMAX_ATTN_H
#define ENTMAX_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ENTMAX_OK = 0,
    ENTMAX_ERR_INVALID = 1,     /* null pointer, bad size, alpha <= 1, workspace too small for ... */
    ENTMAX_ERR_UNSUPPORTED = 2, /* valid but not built: d not in {64, 128}, fp32 backward,
                                   n > 65535 * 128, ...                                         */
    ENTMAX_ERR_ALIGN = 3,       /* a tensor base address is not 16-byte aligned                    */
    ENTMAX_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed                             */
    ENTMAX_ERR_TIMEOUT = 5,     /* a device-side bounded wait ran out (reported by check())        */
    ENTMAX_ERR_WORKSPACE = 6    /* workspace missing or smaller than entmax_attn_workspace_size()  */
} entmax_status;

typedef enum {
    ENTMAX_BF16 = 0, /* bf16 inputs and outputs, fp32 accumulation on the tensor cores (tcgen05) */
    ENTMAX_FP32 = 1  /* fp32 inputs and outputs, fp32 FMA arithmetic throughout (forward only)    */
} entmax_dtype;

/* Device-side counters, accumulated with atomics when opts->stats is non-NULL (zero it first). */
typedef struct {
    unsigned long long rows;             /* query rows solved                                     */
    unsigned long long steps;            /* solver updates of tau after the histogram estimate    */
    unsigned long long fallbacks;        /* updates that were bisection (step left the bracket)   */
    unsigned long long step_hist[9];     /* rows by number of steps, 0..8                         */
    unsigned long long causal_blocks;    /* (query block, key block) pairs with an allowed entry  */
    unsigned long long candidate_blocks; /* pairs the sparse sweeps visited (128-row tiles x 64)  */
    unsigned long long nonzero_blocks;   /* mask bits set                                         */
    unsigned long long sweeps;           /* key sweeps over all tiles (dense + refine + P V)      */
    unsigned long long overflow_rows;    /* rows whose candidates did not fit the on-chip stash   */
    unsigned long long support;          /* nonzero probabilities (entries with z > tau), all rows */
} entmax_stats;

typedef struct {
    float scale;            /* score scale; 0 means 1/sqrt(d)                                      */
    int mask_block;         /* mask block mb (query and key); 0 means 64. bf16: 64; fp32: 32 or 64 */
    int hist_bins;          /* histogram bins B; 0 means 256. Supported: 64, 128, 256              */
    int init_mode;          /* 0: histogram start (default); 1: plain bracket start, no histogram  */
    void* workspace;        /* device scratch, >= entmax_attn_workspace_size() bytes, 256-aligned, */
    size_t workspace_bytes; /* kept by the caller from the forward to the matching backward        */
    entmax_stats* stats;    /* optional device counters, may be NULL                               */
    float* tau_hist;        /* optional device [B,H,n]: the histogram bound tau_h of each row      */
    uint8_t* steps;         /* optional device [B,H,n]: solver steps taken by each row             */
    void* const* events;    /* optional cudaEvent_t handles (as void*) for per-kernel timing, or NULL */
    int num_events;         /* length of `events` (0 when NULL); see "Per-kernel timing" below       */
    void* scratch;          /* optional per-call scratch (>= entmax_attn_scratch_size() bytes, 256-aligned);
                               NULL: the scratch lies inside the workspace (see "Workspace" below)    */
    size_t scratch_bytes;
    float alpha;            /* sizing only: the alpha the workspace will serve (0: any; see below)    */
} entmax_opts;

/* Workspace. The library's device scratch has two parts:
 *   saved   - written by the forward and read by its backward: sum u (fp32 [B,H,n]), the transposed block
 *             mask and, unless the fp16 kernels serve the call (bf16, d = 64, alpha <= 2), U V (fp32
 *             [B,H,n,d]); entmax_attn_saved_size() bytes. The size functions leave U V out only when
 *             opts->alpha names an alpha in (1, 2] (with d = 64, bf16); a workspace sized without U V
 *             makes calls with another alpha return ENTMAX_ERR_WORKSPACE;
 *   scratch - used within one call: the padded per-row delta and row statistic, range words and, for bf16
 *             inputs with d = 64, the fp16 operand copies of Q, K, V, dO; entmax_attn_scratch_size() bytes.
 * With opts->scratch NULL, opts->workspace holds both (entmax_attn_workspace_size() bytes, the sum) and a
 * backward reuses the fp16 copies of Q, K, V that its forward left there. With opts->scratch set,
 * opts->workspace needs only the saved part: only that must be kept from the forward to the backward (the
 * activation memory of the attention is then O, tau, the mask and the saved part), and the backward
 * makes its own fp16 copies in whatever scratch it is given. */

/* Per-kernel timing. When opts->events is set, a call records events[i] on `stream` right before its i-th
 * kernel launch and one more event after its last launch (events past num_events are not recorded; a NULL
 * handle is skipped). The launches of a call, in order:
 *   entmax_attn_fwd, bf16, d = 64, alpha <= 2:  to_f16_pass1, to_f16_pass2, fwd_h, mask_transpose
 *   entmax_attn_fwd, bf16, otherwise:           fwd_tc, mask_transpose
 *   entmax_attn_fwd, fp32:                      fwd_simt
 *   entmax_attn_bwd, d = 64, alpha <= 2:        to_f16_pass1, to_f16_pass2, bwd_pre, bwd_h_dq (keys of unit
 *                                               scale), bwd_h_dq (delta pass, larger keys), bwd_h_dq (larger
 *                                               keys), bwd_h_dkdv: of the three dQ launches, the range of K
 *                                               lets either the first or the other two work; the rest return
 *                                               at once
 *   entmax_attn_bwd, otherwise:                 bwd_pre, bwd_dkdv, bwd_dq
 *   softmax_attn_fwd, d = 64 with a workspace:  to_f16_pass1, to_f16_pass2, softmax_fwd_h
 *   softmax_attn_fwd, otherwise:                softmax_fwd
 *   softmax_attn_bwd, d = 64:                   to_f16_pass1, to_f16_pass2, bwd_pre, bwd_h_dq, bwd_h_dkdv
 *   softmax_attn_bwd, d = 128:                  bwd_pre, bwd_dkdv, bwd_dq
 * The events are recorded by the host thread that makes the call, as part of it; opts->events must stay
 * valid for the duration of the call only. */

/* Bytes of workspace that entmax_attn_fwd/bwd (or softmax_attn_fwd/bwd) need for these sizes, saved and
 * scratch parts together (a single buffer, opts->scratch NULL). Returns 0 for invalid sizes. opts may be
 * NULL (defaults). */
size_t entmax_attn_workspace_size(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* opts);

/* Bytes of the saved part alone (opts->workspace when opts->scratch is set), and of the scratch part
 * (opts->scratch). 0 for invalid sizes. */
size_t entmax_attn_saved_size(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* opts);
size_t entmax_attn_scratch_size(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* opts);

/* Forward. Q, K, V: [B,H,n,d] inputs. O: [B,H,n,d] output (same dtype). tau: float32 [B,H,n]
 * output, the normaliser in z units. block_mask: uint32 output as described above. alpha > 1.
 * causal: 0 or 1. The workspace receives what the backward needs (sum_u, the transposed mask, U V for the
 * bf16 and fp32 kernels and, for bf16 with d = 64 and alpha <= 2, fp16 copies of Q, K, V with their range
 * exponents).
 * fp32 uses the FMA path. bf16 uses the tcgen05 path: with d = 64 and alpha <= 2 on fp16 operand copies
 * (exact for bf16 values of magnitude in [2^-14, 2^15), power-of-two scaled beyond), else on bf16
 * operands with two-term splits. */
entmax_status entmax_attn_fwd(const void* Q, const void* K, const void* V, void* O, float* tau,
                              uint32_t* block_mask, int B, int H, int n, int d, float alpha, int causal,
                              entmax_dtype dt, const entmax_opts* opts, void* stream);

/* Backward (bf16 inputs only). Inputs are the forward's inputs and outputs and dO (bf16 [B,H,n,d]); the
 * workspace must be the one the forward filled, after the same Q, K, V (with d = 64 and alpha <= 2 the
 * backward reads the forward's fp16 copies of them from the workspace). Outputs dQ, dK, dV: float32
 * [B,H,n,d] (fp32 keeps large gradients exact to well below 1e-2; they are accumulated in fp32 TMEM).
 * Visits only the mask's nonzero blocks. */
entmax_status entmax_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                              const float* tau, const uint32_t* block_mask, void* dQ, void* dK, void* dV,
                              int B, int H, int n, int d, float alpha, int causal, entmax_dtype dt,
                              const entmax_opts* opts, void* stream);

/* Dense softmax flash attention in the same library, same tiling: the measurement baseline.
 * lse: float32 [B,H,n] natural-log sum-exp of the scaled scores (output of fwd, input of bwd).
 * With d = 64 and a workspace in opts the forward runs on fp16 operand copies like the entmax forward;
 * without one (opts NULL) it uses the bf16 kernel. */
entmax_status softmax_attn_fwd(const void* Q, const void* K, const void* V, void* O, float* lse,
                               int B, int H, int n, int d, int causal, entmax_dtype dt,
                               const entmax_opts* opts, void* stream);
/* softmax_attn_bwd: dQ, dK, dV float32 like entmax_attn_bwd; needs opts->workspace
 * (softmax_attn_workspace_size() bytes, or any entmax size for the same shape). */
entmax_status softmax_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                               const float* lse, void* dQ, void* dK, void* dV, int B, int H, int n, int d,
                               int causal, entmax_dtype dt, const entmax_opts* opts, void* stream);
/* Bytes of workspace (one buffer) that softmax_attn_fwd/bwd need: the entmax layout without U V
 * (the dense baseline keeps no U V). 0 for invalid sizes. opts may be NULL. */
size_t softmax_attn_workspace_size(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* opts);

/* Forward that allocates nothing and needs no workspace (the paper has no counterpart: this is for
 * callers that cannot allocate device memory, e.g. code running inside a framework that owns the whole
 * device pool, or paths that must not call cudaMalloc, which may synchronise and is not allowed during
 * stream capture). Same arguments, outputs and checks as entmax_attn_fwd; opts may be NULL and any
 * opts->workspace and opts->scratch are ignored. The scratch lives in a 32 MiB (33554432-byte) device array inside the
 * library, which every GPU that loads the library holds until exit; calls whose workspace
 * (entmax_attn_workspace_size) would be larger return ENTMAX_ERR_WORKSPACE. The first call on
 * each device looks up the array's device address (cudaGetSymbolAddress), so make that first call
 * before any stream capture. All calls share the array and it keeps the last call's contents (no part
 * of it needs to start at zero); calls that may overlap on the GPU (other streams, other host threads)
 * race on it, and a later entmax_attn_bwd cannot use it: for training use entmax_attn_fwd. The looked-up address
 * is kept for the life of the process: do not use this entry point after cudaDeviceReset() on that device (the
 * same holds for the device status word behind every entry point). */
entmax_status entmax_attn_fwd_noalloc(const void* Q, const void* K, const void* V, void* O, float* tau,
                                      uint32_t* block_mask, int B, int H, int n, int d, float alpha, int causal,
                                      entmax_dtype dt, const entmax_opts* opts, void* stream);

/* Synchronises `stream`, then returns and clears the device status word of the current device:
 * ENTMAX_ERR_TIMEOUT if a kernel's bounded wait ran out since the last check, ENTMAX_ERR_CUDA if the
 * stream reports an error, else ENTMAX_OK. */
entmax_status entmax_attn_check(void* stream);

/* Test hook for the timeout path: launches one block that waits on a barrier nobody arrives at,
 * with a limit of `limit_us` microseconds (1..2000000), then records ENTMAX_ERR_TIMEOUT and returns. */
entmax_status entmax_attn_selftest_timeout(int limit_us, void* stream);

/* Human-readable name of a status code (static string). */
const char* entmax_status_str(entmax_status s);

/* Library ABI version: 3. Version 2: entmax_opts gained `events`, `num_events`, `scratch`, `scratch_bytes`,
 * `alpha`; entmax_stats gained `support`; entmax_attn_saved_size and entmax_attn_scratch_size were added.
 * Version 3: softmax_attn_workspace_size was added; the scratch part holds fp16 operand copies only for
 * bf16 inputs with d = 64. */
int entmax_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ENTMAX_ATTN_H */
