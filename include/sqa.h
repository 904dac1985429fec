/*
 * sqa.h -- C ABI of the B200 (sm_100a) Sparse Query Attention library.
 *
 * Sparse Query Attention (arXiv 2510.01817, abstract; SQAT-m model card,
 * "Architecture details" and "Model size difference") is scaled dot-product
 * attention with H_q query heads, fewer than the H-way split of the model
 * width, sharing H_kv key/value heads.  The query heads form H_kv contiguous
 * groups of g = H_q / H_kv heads and every head of a group reads the same K and
 * V head (GQA summary, "The idea": one key head and one value head per group;
 * "The notation": GQA-1 is MQA, GQA-H is MHA).  Score FLOPs therefore scale with
 * H_q.  For query head h, kv(h) = floor(h / g):
 *
 *   S_ij  = scale * <Q[b,i,h,:], K[b,j,kv(h),:]>      (-inf where causal and j > i)
 *   lse_i = ln sum_j exp(S_ij)
 *   O_i   = sum_j exp(S_ij - lse_i) V[b,j,kv(h),:]
 *
 * Tensor layouts (all contiguous, row-major, no padding):
 *   q, out, dout, dq : bf16 [B][N][H_q][dh]
 *   k, v, dk, dv     : bf16 [B][N][H_kv][dh]
 *   lse              : fp32 [B][H_q][N], natural log of the sum of exp(scaled scores)
 *
 * Ownership and execution: the caller owns every buffer (device memory, e.g.
 * from PyTorch) and the stream.  Calls are asynchronous on `stream`; the library
 * allocates no device memory at run time and keeps no per-call state on the
 * device, with two exceptions: sqa_bwd_static_scratch works in one file-scope
 * device array that every GPU loading the library holds until exit and that
 * keeps the last call's contents, and the kernels' wait-timeout status words
 * persist until read.  No call synchronises except sqa_device_status and
 * sqa_device_timeout_info, which synchronise the current device to read those
 * words.  Arguments are validated on the host before anything is launched; a
 * call that returns an error has launched nothing.  The calls are thread-safe;
 * error text is kept per host thread.
 */
#ifndef SQA_H_
#define SQA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sqa_stream_t; /* a cudaStream_t; NULL is the legacy default stream */

typedef enum {
    SQA_OK = 0,
    SQA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, H_q not a multiple of H_kv, NaN scale */
    SQA_ERR_UNSUPPORTED = 2, /* head dim not in {16, 32, 64, 128}, g > 128, misaligned pointer, size too large */
    SQA_ERR_CUDA = 3         /* a CUDA runtime/driver call failed; sqa_last_error() has the text */
} sqa_status;

typedef struct {
    int B;    /* batch */
    int N;    /* sequence length (queries and keys) */
    int H_q;  /* query heads */
    int H_kv; /* key/value heads; H_q % H_kv == 0 and H_q / H_kv <= 128 */
    int dh;   /* head dimension: 16, 32, 64 or 128 */
} sqa_shape;

/*
 * Forward pass (the definition above).  q, k, v, out must be 16-byte aligned;
 * lse 4-byte aligned.  out and lse are fully overwritten.  scale <= 0 selects
 * 1/sqrt(dh).  causal != 0 masks keys j > i (the diagonal j == i stays visible).
 */
sqa_status sqa_fwd(const void *q, const void *k, const void *v, void *out, float *lse, sqa_shape s,
                   int causal, float scale, sqa_stream_t stream);

/*
 * Bytes of device scratch that sqa_fwd_with_workspace uses for shape s: 0 for
 * every shape except small ones (dh <= 64, B * H_kv * ceil(N / T) Q tiles of
 * T = floor(128 / g) tokens filling less than half the device's SMs), whose
 * key tiles are then split into ranges run by separate CTAs: per range and
 * stacked row, dh + 1 fp32 partial values, and one int counter per stacked row.
 * The answer depends on the SM count of the current device (148 when none can
 * be queried).
 */
size_t sqa_fwd_workspace_bytes(sqa_shape s, int causal);

/*
 * sqa_fwd with scratch (same definition, arguments and results).  With
 * sqa_fwd_workspace_bytes(s, causal) > 0, workspace (256-byte aligned, at least
 * that many bytes, contents arbitrary) takes the ranges' partial outputs and
 * log-sum-exps; each row's ranges are merged by the CTA that finishes the last
 * of them (its counter, cleared by an asynchronous memset on `stream` before the
 * kernel, says which).  The partials are normalised within their range, so the
 * merge is O = sum_c 2^(L_c - M) O_c / sum_c 2^(L_c - M) in fp32.  With 0 bytes
 * needed, workspace may be NULL and the call is sqa_fwd.  Errors: those of
 * sqa_fwd; SQA_ERR_INVALID_ARG for a null or too small workspace when one is
 * needed, SQA_ERR_UNSUPPORTED for a misaligned one.  The workspace must not be
 * used by another call until this one has completed on `stream`.
 */
sqa_status sqa_fwd_with_workspace(const void *q, const void *k, const void *v, void *out, float *lse,
                                  void *workspace, size_t workspace_bytes, sqa_shape s, int causal,
                                  float scale, sqa_stream_t stream);

/*
 * Bytes of device scratch that sqa_bwd needs for shape s (fp32 dQ accumulator
 * plus per-row softmax statistics).  The caller allocates it; 256-byte aligned.
 */
size_t sqa_bwd_workspace_bytes(sqa_shape s);

/*
 * Backward pass of L = sum(dout * out) through the forward above.
 * Inputs: dout, q, k, v, out (bf16, the forward's output) and lse (fp32, the
 * forward's).  Outputs: dq (bf16, [B][N][H_q][dh]), dk and dv (bf16,
 * [B][N][H_kv][dh]); all three are fully overwritten.  dK and dV of a key/value
 * head sum the contributions of every query head in its group.
 *   D_i   = <dO_i, O_i>,  P_ij = exp(S_ij - lse_i),  dP_ij = <dO_i, V_j>
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij K_j;  dK_j = scale sum_{h in group} sum_i dS_ij Q_i;
 *   dV_j  = sum_{h in group} sum_i P_ij dO_i
 * workspace must hold sqa_bwd_workspace_bytes(s) bytes and be 256-byte
 * aligned; its contents on entry do not matter and are clobbered.
 */
sqa_status sqa_bwd(const void *dout, const void *q, const void *k, const void *v, const void *out,
                   const float *lse, void *dq, void *dk, void *dv, void *workspace,
                   size_t workspace_bytes, sqa_shape s, int causal, float scale,
                   sqa_stream_t stream);

/*
 * Largest scratch, in bytes, that sqa_bwd_static_scratch can use (64 MiB).
 */
#define SQA_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * sqa_bwd without a workspace argument, for callers that cannot allocate
 * device memory: a plugin inside a framework that owns every device
 * allocation (a cudaMalloc there bypasses the framework's pool and can
 * synchronise the whole device), or code that must not allocate once a step
 * has started.  The paper has no counterpart to this entry point.
 *
 * Arguments, layouts, results and errors are those of sqa_bwd.  The scratch
 * that sqa_bwd takes from the caller lives here in one file-scope device array
 * of SQA_STATIC_SCRATCH_BYTES, which every GPU that loads the library holds
 * until the process exits; shapes whose sqa_bwd_workspace_bytes() exceeds it
 * are rejected with SQA_ERR_UNSUPPORTED before anything is launched.  Nothing
 * is allocated or freed by this call.
 *
 * Every call made outside a stream capture looks up the array's device
 * address on the current device (so a context torn down and rebuilt between
 * calls, e.g. by cudaDeviceReset, leaves no stale pointer); a call made while
 * `stream` is capturing uses the address found by the last call outside a
 * capture on that device, and fails with SQA_ERR_INVALID_ARG if there was
 * none.  So make a first call on each device before any stream capture.  All
 * calls share the one array and it keeps the last call's contents; the
 * kernels clear what must start at zero.  Calls whose GPU work overlaps (on
 * different streams, or from different threads) race on the array: order them.
 */
sqa_status sqa_bwd_static_scratch(const void *dout, const void *q, const void *k, const void *v,
                                  const void *out, const float *lse, void *dq, void *dk, void *dv,
                                  sqa_shape s, int causal, float scale, sqa_stream_t stream);

/*
 * The full SQA layer around the attention core (SQAT-m model card, "Model size
 * difference": the query and output projections shrink with the query-head
 * count; "Architecture details": rotary position embedding):
 *
 *   [Q | K | V] = X W_qkv,   Q, K turned by the rotary embedding,
 *   O = the attention core above (sqa_fwd),   Y = O W_o
 *
 * with no biases.  Layouts (row-major, contiguous, bf16 unless noted;
 * M = B * N tokens, W = (H_q + 2 H_kv) * dh):
 *   x, y, dy, dx : [B][N][d]
 *   w_qkv        : [d][W]; columns [0, H_q dh) are W_q (query head h in
 *                  columns h dh .. h dh + dh - 1), then H_kv dh columns of W_k,
 *                  then H_kv dh columns of W_v
 *   w_o          : [H_q dh][d]
 *   q, out       : [B][N][H_q][dh];  k, v : [B][N][H_kv][dh];  lse fp32 [B][H_q][N]
 *                  (the rotated projections and the core's outputs, as sqa_fwd
 *                  takes and gives them; the backward needs them)
 *   dw_qkv, dw_o : fp32, the shapes of w_qkv and w_o
 * Rotary embedding: channels (2j, 2j+1) of every query and key head of the
 * token at position i = token index within its sequence turn by the angle
 * i * rope_base^(-2j/dh) (cos/sin formed in double precision, rounded to
 * fp32); rope_base = 0 leaves Q and K unrotated.  d must be a multiple of 8;
 * the other limits are sqa_fwd's.
 */
typedef struct {
    int B, N;           /* batch, tokens per sequence */
    int d;              /* model width */
    int H_q, H_kv, dh;  /* as in sqa_shape */
} sqa_layer_shape;

/*
 * Bytes of device scratch that sqa_layer_fwd (backward = 0) or sqa_layer_bwd
 * (backward != 0) needs; 0 if the shape is invalid.  The caller allocates it,
 * 256-byte aligned; its contents on entry do not matter.
 */
size_t sqa_layer_workspace_bytes(sqa_layer_shape s, int backward);

/*
 * Layer forward: writes y and the saved tensors q, k, v (rotated), out and lse.
 * Three kernels on `stream` (a tcgen05 GEMM with the rotation in its epilogue,
 * the attention core, the output GEMM), plus a small table kernel when
 * rope_base > 0.  causal and scale as for sqa_fwd.  Errors as for sqa_fwd,
 * returned before any launch; SQA_ERR_INVALID_ARG for a workspace smaller
 * than sqa_layer_workspace_bytes(s, 0) or a negative or non-finite rope_base.
 */
sqa_status sqa_layer_fwd(const void *x, const void *w_qkv, const void *w_o, void *y, void *q, void *k,
                         void *v, void *out, float *lse, void *workspace, size_t workspace_bytes,
                         sqa_layer_shape s, int causal, float scale, float rope_base,
                         sqa_stream_t stream);

/*
 * Layer backward of L = sum(dy * y): dx (bf16) and the weight gradients dw_qkv
 * and dw_o (fp32, fully overwritten).  Takes the forward's x, weights and saved
 * tensors.  Steps: dO = dY W_o^T; dW_o = O^T dY; the core backward (sqa_bwd)
 * gives dQ, dK, dV of the rotated projections; the rotation is undone on dQ
 * and dK; dW_qkv = X^T [dQ | dK | dV]; dX = [dQ | dK | dV] W_qkv^T.  The
 * weight-gradient products reduce over all M tokens with fp32 reductions in a
 * run-dependent order.  workspace: sqa_layer_workspace_bytes(s, 1) bytes.
 */
sqa_status sqa_layer_bwd(const void *dy, const void *x, const void *w_qkv, const void *w_o, const void *q,
                         const void *k, const void *v, const void *out, const float *lse, void *dx,
                         float *dw_qkv, float *dw_o, void *workspace, size_t workspace_bytes,
                         sqa_layer_shape s, int causal, float scale, float rope_base,
                         sqa_stream_t stream);

/*
 * One SQAT-m decoder block (SQAT-m model card, "Architecture details": SQA,
 * RoPE, RMS Norm and a SwiGLU feed-forward of hidden width 768), read as the
 * plain pre-norm residual block with no biases:
 *
 *   n1 = RMSNorm(x; g1),  h = x + SQA layer(n1),
 *   n2 = RMSNorm(h; g2),  y = h + (silu(n2 W1) * (n2 W3)) W2,
 *   RMSNorm(x; g) = g * x / sqrt(mean over the d features of x^2 + 1e-6),
 *   silu(a) = a / (1 + e^-a).
 *
 * Weights (bf16): g1, g2 [d]; w_qkv, w_o as for sqa_layer_fwd; w1, w3
 * [d][hidden]; w2 [hidden][d].  x, y, dy, dx: bf16 [B][N][d].  Gradients
 * (fp32, fully overwritten; the weight gradients reduce over all tokens in a
 * run-dependent order) have the weights' shapes.  Every activation the
 * backward needs (the normalised rows and their 1/RMS, the layer's q, k, v,
 * core output and lse, h, the feed-forward's a = n2 W1, b = n2 W3 and
 * silu(a) * b, all bf16 but the statistics) is kept in `state`, which the
 * forward writes and the backward reads, plus the backward's scratch: the
 * caller allocates sqa_block_state_bytes(s) bytes, 256-byte aligned, and keeps
 * it between the two calls.  Additional limits: hidden a multiple of 8,
 * d <= 8192.
 */
typedef struct {
    int B, N, d, H_q, H_kv, dh;
    int hidden; /* feed-forward width */
} sqa_block_shape;

typedef struct {
    const void *g1, *w_qkv, *w_o, *g2, *w1, *w3, *w2;
} sqa_block_weights;

typedef struct {
    float *g1, *w_qkv, *w_o, *g2, *w1, *w3, *w2;
} sqa_block_grads;

/* Bytes of the forward-to-backward state of one block; 0 if s is invalid. */
size_t sqa_block_state_bytes(sqa_block_shape s);

/*
 * Block forward: y, and the saved activations in `state`.  causal, scale and
 * rope_base as for sqa_layer_fwd.  Errors as for sqa_layer_fwd, returned
 * before any launch.
 */
sqa_status sqa_block_fwd(const void *x, const sqa_block_weights *w, void *y, void *state, size_t state_bytes,
                         sqa_block_shape s, int causal, float scale, float rope_base, sqa_stream_t stream);

/*
 * Block backward of L = sum(dy * y), after sqa_block_fwd on the same x,
 * weights and state: dx and every gradient in *grads.  Steps: dM = dY W2^T
 * with da = dM b silu'(a), db = dM silu(a) in the same product's epilogue;
 * dW2 = m^T dY, dW1 = n2^T da, dW3 = n2^T db; dn2 = da W1^T + db W3^T;
 * dh = dY + RMSNorm'(h) dn2 (and dg2); the layer's backward (sqa_layer_bwd)
 * with X = n1 and dY = dh; dx = dh + RMSNorm'(x) dn1 (and dg1).
 */
sqa_status sqa_block_bwd(const void *dy, const void *x, const sqa_block_weights *w, void *state,
                         size_t state_bytes, void *dx, const sqa_block_grads *grads, sqa_block_shape s,
                         int causal, float scale, float rope_base, sqa_stream_t stream);

/* Static text for a status code. */
const char *sqa_status_string(sqa_status status);

/* Detail of the last error on the calling host thread ("" if none). */
const char *sqa_last_error(void);

/*
 * Device-side wait status.  Every wait inside the kernels gives up after about
 * two seconds, sets a bit in a per-device status word and lets the kernel end,
 * so a broken pipeline reports an error instead of hanging the GPU.  This call
 * synchronises the current device, returns the word (0 = no timeout seen) and,
 * if clear != 0, resets it.  Returns SQA_ERR_CUDA if it could not be read.
 */
sqa_status sqa_device_status(unsigned int *word, int clear);

/*
 * Where the first wait that gave up on the current device was: info[0] = 1 if
 * one did (0 otherwise), info[1] = block index, info[2] = (role << 16) |
 * barrier index within the kernel's barrier block (roles: 0 producer, 1 MMA
 * issuer, 2 softmax, 3 epilogue or converter, 4 drain), info[3] = (thread << 8)
 * | phase parity.  Synchronises the device; clear != 0 resets the record.
 */
sqa_status sqa_device_timeout_info(unsigned int info[4], int clear);

/*
 * Optional timing hook for benchmarks.  While set on the calling host thread,
 * sqa_fwd (kernel = 0), sqa_bwd (kernel = 1) or sqa_decode (kernel = 2, its
 * split kernel) records `start` on its stream just before launching its main
 * attention kernel and `stop` just after it, so
 * the caller can time that one kernel with cudaEventElapsedTime.  start and
 * stop are cudaEvent_t handles owned by the caller; pass NULL for both to turn
 * the hook off.  Returns SQA_ERR_INVALID_ARG for another kernel index or when
 * only one of the two events is given.
 */
sqa_status sqa_set_timing_events(int kernel, void *start, void *stop);

/*
 * Bytes of device scratch that sqa_decode needs for shape s, 0 if s is
 * invalid.  The caller allocates it; 256-byte aligned.
 */
size_t sqa_decode_workspace_bytes(sqa_shape s);

/*
 * Decoding step: one new
 * query token per sequence attends to the first seq_lens[b] entries of its
 * key/value cache, with no further mask (arXiv 2510.01817 abstract: SQA
 * reduces query heads, so this memory-bound step costs what GQA's does; GQA
 * summary, "The idea": the K/V head count sets the cache size).
 *
 *   s_j   = scale * <q[b,h,:], K[b,j,kv(h),:]>,  j < seq_lens[b]
 *   lse   = ln sum_j exp(s_j),  out[b,h,:] = sum_j exp(s_j - lse) V[b,j,kv(h),:]
 *
 * Shapes (s.N is the cache capacity):
 *   q, out           : bf16 [B][H_q][dh]
 *   k_cache, v_cache : bf16 [B][N][H_kv][dh], 16-byte aligned
 *   seq_lens         : int32 [B] on the device, or NULL for all N; values are
 *                      clamped to [0, N]; a length of 0 gives out = 0 and
 *                      lse = -inf
 *   lse              : fp32 [B][H_q]
 *   workspace        : sqa_decode_workspace_bytes(s) bytes, 256-byte aligned,
 *                      contents ignored and overwritten
 * Supported: dh in {16, 32, 64, 128}, H_q / H_kv <= 128, B * H_kv <= 65535.
 * Two kernels on `stream`, asynchronous, nothing allocated; out and lse are
 * fully overwritten.  Errors as for sqa_fwd, returned before any launch.
 */
sqa_status sqa_decode(const void *q, const void *k_cache, const void *v_cache, const int *seq_lens,
                      void *out, float *lse, void *workspace, size_t workspace_bytes, sqa_shape s,
                      float scale, sqa_stream_t stream);

/*
 * Self-test hook for the polynomial exponential that sqa_fwd uses for part of
 * the softmax exponentials at dh <= 32 (2 of every 8 pairs of scores in tiles
 * without masked keys; the rest use the special-function unit).  It exists so
 * that tests can compare that function with 2^x; the pages have no
 * counterpart.  y[i] = the library's 2^x[i] for 0 <= i < n; x and y are device
 * pointers to fp32 arrays of n elements, 8-byte aligned, owned by the caller.
 * Method: n = round(x), f = x - n, a degree-3 minimax polynomial in f (largest
 * relative error 7.5e-5), exponent n added to its bits; x is clamped to -126
 * first, so results below 2^-126 come out as about 1.2e-38.  Asynchronous on
 * `stream`; n <= 0 launches nothing.  SQA_ERR_INVALID_ARG for null or
 * misaligned pointers.
 */
sqa_status sqa_selftest_exp2_poly(const float *x, float *y, int n, sqa_stream_t stream);

/*
 * Throughput probe of the special-function unit's exponential (ex2.approx,
 * the instruction the softmax uses for 2^x), behind the exp2 roofline that the
 * dh <= 32 kernels are measured against; the pages have no counterpart.
 * Launches n_blocks blocks of 256 threads on `stream`; every thread runs 8
 * independent chains of `iters` dependent exponentials (8 * iters per thread)
 * and writes one float (the chains' sum, so nothing is optimised away) to
 * out[block * 256 + thread].  out: device fp32 array of n_blocks * 256
 * elements, owned by the caller.  The caller times the launch (events on the
 * stream).  SQA_ERR_INVALID_ARG for a null `out`, n_blocks outside 1..65535 or
 * iters outside 1..1048576, before any launch.
 */
sqa_status sqa_selftest_exp2_rate(float *out, int n_blocks, int iters, sqa_stream_t stream);

/*
 * Self-test hook for the kernels' bounded waits, so that tests can exercise
 * the failure path without faulting or hanging a GPU; the pages have no
 * counterpart.  Launches one small kernel on `stream` whose thread waits on an
 * mbarrier that nothing ever completes, through the same bounded wait the
 * attention kernels use, but giving up after limit_us microseconds (1 to
 * 100000) instead of about two seconds.  It then sets bit `site` (0 to 4, the
 * roles of sqa_device_timeout_info) in the device status word, records itself
 * in the timeout record if that is empty (block 0, thread 0, parity 0) and
 * returns; the context stays usable.  SQA_ERR_INVALID_ARG for limits or sites
 * out of range, before any launch.
 */
sqa_status sqa_selftest_wait_timeout(unsigned int limit_us, unsigned int site, sqa_stream_t stream);

/* Library version as an integer (major * 10000 + minor * 100 + patch). */
int sqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SQA_H_ */
