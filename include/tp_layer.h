/*
 * tp_layer.h -- C ABI of the B200 (sm_100a) tensor-parallel transformer
 * sublayer library (libtplayer.so).
 *
 * The method is Megatron-LM's intra-layer (tensor) model parallelism
 * (Shoeybi et al., 2019), as described on the pages
 *   "Megatron-LM: what the tensor parallelism paper actually says"
 *     - "How transformer layers actually decompose"  (MLP: W1 column split,
 *       local GeLU, W2 row split, partial outputs summed),
 *     - "The attention heads split" (Q/K/V split by head, local attention,
 *       row-split output projection, partial outputs summed),
 *     - "The layernorm placement the paper flags as critical" (pre-LN);
 *   "Megatron-LM interactive explainer" - "One Idea, Two Insertions" (one
 *       reduction in the forward and one in the backward of each pair).
 * All t shards run on ONE GPU: the cross-shard all-reduce of the forward is
 * the fp32 accumulation of the t partial products inside the row-parallel
 * GEMM, and the backward reduction of input gradients is the same walk in
 * the input-gradient GEMM.  No collective is issued.
 *
 * Conventions for every entry point
 *  - Element type: bf16, passed as raw 16-bit patterns (tp_bf16); fp16 or fp32
 *    where stated.  Accumulation is fp32; outputs are rounded to nearest even once.
 *  - Pointers: DEVICE pointers owned by the caller, 16-byte aligned, dense
 *    row-major, unless stated otherwise.  The library allocates nothing on the
 *    compute path.  Its only state: cached per-device attributes and kernel
 *    settings, one device error word per device (tp_check_error), the
 *    optional launch trace (tp_trace_begin) and the static scratch array of
 *    tp_layernorm_bwd_noalloc.
 *  - Shapes: T = batch*seq tokens (batch outer), D = hidden, F = ffn,
 *    H = heads, dh = head_dim (D = H*dh), t = tensor-parallel degree,
 *    Ft = F/t, Dt = D/t.  Activations x, y: [T][D].
 *  - Shard-packed weights (each shard's block contiguous, the way one GPU
 *    of a t-GPU group would hold it; tp_shard_* convert):
 *      W1   [t][D][Ft]    column shards of W1 [D][F]
 *      W2   [t][Ft][D]    row shards of W2 [F][D] (byte-identical to W2)
 *      Wqkv [t][D][3*Dt]  shard i = [Wq_i | Wk_i | Wv_i], the columns of heads
 *                         i*H/t .. (i+1)*H/t-1 of Wq, Wk, Wv [D][D]
 *      Wout [t][Dt][D]    row shards of Wout [D][D]
 *    Biases follow their matrix: b1 [t][Ft], bqkv [t][3*Dt], b2/bout [D].
 *    The bias of a row-parallel product is added once, after the shard sum.
 *  - Streams: every call only enqueues work on `stream` (a cudaStream_t, or
 *    NULL for the legacy default stream) and returns; it never synchronises.
 *  - Errors: no exception crosses the ABI.  Arguments are validated on the
 *    host before anything is launched; on failure nothing is enqueued and a
 *    status != TP_OK is returned.  Launch failures return TP_ERR_CUDA.  A
 *    device-side wait that exceeds its bound (about 2 s) records a code in
 *    the library's device error word and the kernel returns early; read it
 *    with tp_check_error after synchronising.
 */
#ifndef TP_LAYER_H
#define TP_LAYER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t tp_bf16;  /* raw bfloat16 bits */
typedef uint16_t tp_f16;   /* raw IEEE binary16 (fp16) bits: the buffers inside the attention
                              sublayer that hold fp16, never bf16 (qkv, LN1's output u1) */
typedef void* tp_stream;   /* cudaStream_t */

typedef enum {
  TP_OK = 0,
  TP_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, t not dividing H or F, D != H*dh */
  TP_ERR_UNSUPPORTED = 2,  /* valid but not provided: t not in {1,2,4,8}, dh not in {64,128},
                              batch*seq >= 2^31, layer entry points with hidden > 8192 */
  TP_ERR_MISALIGNED = 3,   /* pointer not 16-byte aligned or a row not a multiple of 8 elements */
  TP_ERR_WORKSPACE = 4,    /* workspace pointer null or smaller than tp_workspace_size */
  TP_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed */
  TP_ERR_TIMEOUT = 6,      /* a bounded device wait expired (from tp_check_error) */
  TP_ERR_RANGE = 7         /* a value stored as fp16 exceeded +-65504 (from tp_check_error) */
} tp_status;

/* Codes of the device error word (read by tp_check_error):
 *   0x0F1          the bounded-wait self-test (tp_selftest_wait_timeout)     -> TP_ERR_TIMEOUT
 *   0x101 - 0x1FF  a GEMM kernel's wait expired                              -> TP_ERR_TIMEOUT
 *   0x201 - 0x2FF  an attention kernel's wait expired                        -> TP_ERR_TIMEOUT
 *   0x301          a value written as fp16 (qkv, u1, dO, dqkv, the fp16
 *                  copies of x or Wqkv) was beyond the fp16 range; it is
 *                  stored as +-inf and everything computed from it is
 *                  meaningless                                               -> TP_ERR_RANGE
 * The word keeps the first code recorded since it was last cleared. */

/* Sizes of one problem.  Fields an operation does not use are ignored
 * (e.g. heads/head_dim for the MLP, ffn for attention). */
typedef struct {
  int batch;     /* B >= 0 */
  int seq;       /* S >= 0; T = B*S < 2^31.  T = 0 is an empty problem: nothing is
                    computed, parameter gradients are zeroed, and activation
                    pointers may be NULL */
  int hidden;    /* D, multiple of 8*t */
  int ffn;       /* F, multiple of 8*t */
  int heads;     /* H, multiple of t */
  int head_dim;  /* dh in {64, 128}, D = H*dh */
  int t;         /* tensor-parallel degree in {1, 2, 4, 8} */
  int causal;    /* attention mask: 1 = key s' visible to query s iff s' <= s; 0 = none */
  float ln_eps;  /* LayerNorm epsilon (layer entry points only), > 0 */
} tp_dims;

typedef enum {
  TP_OP_MLP_FWD = 0,
  TP_OP_MLP_BWD = 1,
  TP_OP_ATTN_FWD = 2,
  TP_OP_ATTN_BWD = 3,
  TP_OP_LAYER_FWD = 4,
  TP_OP_LAYER_BWD = 5,
  TP_OP_POSTLN_FWD = 6,
  TP_OP_POSTLN_BWD = 7,
  TP_OP_LAYER_FWD_NOSAVE = 8,
  TP_OP_LAYER_BWD_RECOMPUTE = 9
} tp_op;

/* Version string of the library. */
const char* tp_version(void);

/* Human-readable name of a status code (static storage). */
const char* tp_status_string(tp_status s);

/* Bytes of device workspace operation `op` needs for `dims` (0 if none, or
 * if the dims are invalid).  The workspace is scratch: its contents on entry
 * are ignored and on return are unspecified.  Calls that may run at the same
 * time need distinct workspaces. */
size_t tp_workspace_size(int op, const tp_dims* dims);

/* Synchronises the current device, then reads and clears the library's
 * device error word.  The code (0 if none) is stored in *code if code != NULL.
 * TP_ERR_RANGE for code 0x301 (an fp16 overflow), TP_ERR_TIMEOUT for any
 * other nonzero code (a bounded wait expired), TP_ERR_CUDA if the
 * synchronisation or the read failed, TP_OK otherwise. */
tp_status tp_check_error(unsigned int* code);

/* ------------------------------------------------------------------ layout
 * Slicing exactly as "How transformer layers actually decompose" and "The
 * attention heads split" define it; bit-exact copies.  All on device,
 * enqueued on `stream`; `src` and `dst` must not overlap. */

/* W [rows][cols] -> [t][rows][cols/t]; shard i holds columns i*cols/t .. (i+1)*cols/t-1. */
tp_status tp_shard_cols(const tp_bf16* w, int rows, int cols, int t, tp_bf16* out, tp_stream stream);
/* Inverse of tp_shard_cols. */
tp_status tp_unshard_cols(const tp_bf16* packed, int rows, int cols, int t, tp_bf16* w, tp_stream stream);
/* W [rows][cols] -> [t][rows/t][cols]; shard i holds rows i*rows/t .. (i+1)*rows/t-1.
 * The packed layout is byte-identical to W; this is a copy. */
tp_status tp_shard_rows(const tp_bf16* w, int rows, int cols, int t, tp_bf16* out, tp_stream stream);
/* Inverse of tp_shard_rows (a copy). */
tp_status tp_unshard_rows(const tp_bf16* packed, int rows, int cols, int t, tp_bf16* w, tp_stream stream);
/* Fused QKV matrix (or bias, rows = 1) [rows][3*hidden] = [Wq | Wk | Wv] ->
 * [t][rows][3*hidden/t], shard i = [Wq_i | Wk_i | Wv_i] holding the columns of
 * heads i*heads/t .. (i+1)*heads/t-1.  heads % t == 0 and hidden % heads == 0. */
tp_status tp_shard_qkv_heads(const tp_bf16* w, int rows, int hidden, int heads, int t, tp_bf16* out,
                             tp_stream stream);
/* Inverse of tp_shard_qkv_heads. */
tp_status tp_unshard_qkv_heads(const tp_bf16* packed, int rows, int hidden, int heads, int t,
                               tp_bf16* w, tp_stream stream);

/* ------------------------------------------------------------------ MLP
 * "How transformer layers actually decompose": output = GeLU(x W1) W2 with
 * W1 split by columns and W2 by rows; GeLU is the tanh form
 * 0.5 a (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3))).
 *
 * tp_mlp_fwd:
 *   a_save[i] = x W1_i + b1_i             [t][T][Ft]   (pre-activation, saved)
 *   h_save[i] = GeLU(a_save[i])          [t][T][Ft]   (activation, saved)
 *   y = sum_{i=0..t-1} h_save[i] W2_i + b2 (+ resid)   [T][D]
 * The shard sum is accumulated in fp32 in shard order and rounded once.
 * b1, b2, resid may be NULL (zero).  Uses dims: batch, seq, hidden, ffn, t.
 * No workspace (pass NULL, 0). */
tp_status tp_mlp_fwd(const tp_dims* dims, const tp_bf16* x, const tp_bf16* w1, const tp_bf16* b1,
                     const tp_bf16* w2, const tp_bf16* b2, const tp_bf16* resid, tp_bf16* y,
                     tp_bf16* a_save, tp_bf16* h_save, void* ws, size_t ws_bytes, tp_stream stream);

/* tp_mlp_bwd: vector-Jacobian product of tp_mlp_fwd for upstream gradient dy [T][D]:
 *   dA_i  = (dy W2_i^T) * GeLU'(a_save[i])          (workspace)
 *   dw2_i = h_save[i]^T dy       [t][Ft][D]
 *   dw1_i = x^T dA_i             [t][D][Ft]
 *   dx    = sum_i dA_i W1_i^T (+ dres)   [T][D]     (backward shard reduction)
 *   db1   = column sums of dA [t][Ft], db2 = column sums of dy [D]
 * dres (the gradient arriving through a residual branch) and db1/db2 may be
 * NULL.  Workspace: tp_workspace_size(TP_OP_MLP_BWD, dims) bytes. */
tp_status tp_mlp_bwd(const tp_dims* dims, const tp_bf16* x, const tp_bf16* w1, const tp_bf16* w2,
                     const tp_bf16* a_save, const tp_bf16* h_save, const tp_bf16* dy,
                     const tp_bf16* dres, tp_bf16* dx, tp_bf16* dw1, tp_bf16* dw2, tp_bf16* db1,
                     tp_bf16* db2, void* ws, size_t ws_bytes, tp_stream stream);

/* ------------------------------------------------------------------ attention
 * "The attention heads split": shard i owns heads i*H/t .. (i+1)*H/t-1.
 *
 * tp_attn_fwd:
 *   qkv_save[i] = x Wqkv_i + bqkv_i        [t][T][3*Dt], fp16 (tp_f16); within shard i,
 *                 columns [0,Dt) are q, [Dt,2Dt) k, [2Dt,3Dt) v, local head j at j*dh
 *   per head:  O = softmax(q k^T / sqrt(dh) + mask) v, softmax in fp32;
 *              lse_save = log-sum-exp of the scaled masked scores, fp32 [B][H][S]
 *   o_save[i]   = the shard's head outputs  [t][T][Dt] (bf16)
 *   y = sum_i o_save[i] Wout_i + bout (+ resid)      [T][D]
 * Inside the attention sublayer the products run on fp16 operands (x and Wqkv
 * are converted, q/k/v, P, dO, dS are fp16; fp32 accumulation): with bf16
 * storage the softmax over long causal rows amplifies the rounding of q and k
 * to a relative error near 6e-3 in O at S = 2048, with fp16 near 2e-3.  A value
 * beyond the fp16 range (|v| > 65504) sets device error code 0x301
 * (tp_check_error reports TP_ERR_RANGE with that code).
 * bqkv, bout, resid may be NULL.  Uses batch, seq, hidden, heads, head_dim, t,
 * causal.  Workspace: tp_workspace_size(TP_OP_ATTN_FWD, dims) bytes. */
tp_status tp_attn_fwd(const tp_dims* dims, const tp_bf16* x, const tp_bf16* wqkv,
                      const tp_bf16* bqkv, const tp_bf16* wout, const tp_bf16* bout,
                      const tp_bf16* resid, tp_bf16* y, tp_f16* qkv_save, tp_bf16* o_save,
                      float* lse_save, void* ws, size_t ws_bytes, tp_stream stream);

/* tp_attn_bwd: vector-Jacobian product of tp_attn_fwd for dy [T][D]:
 *   dO_i = dy Wout_i^T; dwout_i = o_save[i]^T dy   [t][Dt][D]
 *   per head: dv = P^T dO, dP = dO v^T, dS = P * (dP - rowsum(dO * O)),
 *             dq = dS k / sqrt(dh), dk = dS^T q / sqrt(dh)     (P recomputed from lse)
 *   dwqkv_i = x^T dqkv_i  [t][D][3*Dt];  dx = sum_i dqkv_i Wqkv_i^T (+ dres)
 *   dbqkv = column sums of dqkv [t][3*Dt], dbout = column sums of dy [D]
 * dres, dbqkv, dbout may be NULL.  Workspace: tp_workspace_size(TP_OP_ATTN_BWD). */
tp_status tp_attn_bwd(const tp_dims* dims, const tp_bf16* x, const tp_bf16* wqkv,
                      const tp_bf16* wout, const tp_f16* qkv_save, const tp_bf16* o_save,
                      const float* lse_save, const tp_bf16* dy, const tp_bf16* dres, tp_bf16* dx,
                      tp_bf16* dwqkv, tp_bf16* dbqkv, tp_bf16* dwout, tp_bf16* dbout, void* ws,
                      size_t ws_bytes, tp_stream stream);

/* tp_attn_set_ds_limit: how the attention backward forms dq = dS k.  When the
 * fp16 array dS^T of all heads, B*H*S_pad*S_pad*2 bytes with S_pad = seq
 * rounded up to 128, takes at most max_bytes, the kernel that forms dk and dv
 * also stores dS^T in the workspace and the dq kernel reads it back; above the
 * limit the dq kernel recomputes the scores q k^T and dP = dO v^T from the
 * saved lse instead.  The two give dq equal up to fp32 rounding order.  The
 * limit is process-wide, 4 GiB by default (0: always recompute), and enters
 * tp_workspace_size and tp_rank_workspace_size for TP_OP_ATTN_BWD and the
 * layer backward ops: size workspaces after setting it (a smaller workspace
 * gives TP_ERR_WORKSPACE).  A call already running keeps the value it read
 * when it started, so setting the limit from another thread never changes
 * the workspace a running call expects.  Returns the previous limit.  Not an operation of the pages: a choice of
 * how to run the backward of their attention. */
size_t tp_attn_set_ds_limit(size_t max_bytes);

/* ------------------------------------------------------------------ pre-LN layer
 * "The layernorm placement the paper flags as critical":
 *   h = x + Attn(LN1(x));  y = h + MLP(LN2(h))
 * LayerNorm: biased variance over D, eps = dims->ln_eps, affine gamma/beta
 * (bf16); mean and rstd saved in fp32.  Dropout is not applied. */
typedef struct {
  const tp_bf16 *ln1_g, *ln1_b;   /* [D] */
  const tp_bf16 *wqkv, *bqkv;     /* [t][D][3Dt], [t][3Dt] (bqkv may be NULL) */
  const tp_bf16 *wout, *bout;     /* [t][Dt][D], [D] (bout may be NULL) */
  const tp_bf16 *ln2_g, *ln2_b;   /* [D] */
  const tp_bf16 *w1, *b1;         /* [t][D][Ft], [t][Ft] (b1 may be NULL) */
  const tp_bf16 *w2, *b2;         /* [t][Ft][D], [D] (b2 may be NULL) */
} tp_layer_params;

/* Activations saved by tp_layer_fwd for tp_layer_bwd (all caller-owned). */
typedef struct {
  tp_f16* u1;             /* LN1(x) [T][D], fp16 (it feeds only the fp16 attention products) */
  float *mean1, *rstd1;   /* [T] */
  tp_f16* qkv;            /* [t][T][3Dt], fp16 */
  tp_bf16* o;             /* [t][T][Dt] */
  float* lse;             /* [B][H][S] */
  tp_bf16* h;             /* x + attention output [T][D] */
  tp_bf16* u2;            /* LN2(h) [T][D] */
  float *mean2, *rstd2;   /* [T] */
  tp_bf16* a;             /* MLP pre-activation [t][T][Ft] */
  tp_bf16* hact;          /* MLP activation [t][T][Ft] */
  tp_f16* wqkv16;         /* optional (may be NULL): [t][D][3Dt] fp16 copy of params->wqkv.
                             tp_layer_fwd writes it and tp_layer_bwd reads it instead of
                             converting Wqkv again; the weights must not change between the
                             two calls.  NULL: each call converts into its workspace. */
} tp_layer_acts;

/* Parameter gradients written by tp_layer_bwd (same layouts as the parameters;
 * any bias / LayerNorm gradient pointer may be NULL to skip it). */
typedef struct {
  tp_bf16 *dln1_g, *dln1_b, *dwqkv, *dbqkv, *dwout, *dbout;
  tp_bf16 *dln2_g, *dln2_b, *dw1, *db1, *dw2, *db2;
} tp_layer_grads;

/* tp_layer_fwd: x [T][D] -> y [T][D], filling every field of *acts.
 * Workspace: tp_workspace_size(TP_OP_LAYER_FWD, dims) bytes. */
tp_status tp_layer_fwd(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* params,
                       const tp_layer_acts* acts, tp_bf16* y, void* ws, size_t ws_bytes,
                       tp_stream stream);

/* tp_layer_bwd: dy [T][D] -> dx [T][D] and *grads, from the activations that
 * tp_layer_fwd saved for the same x and params.
 *   dh = dy + LN2^T(MLP^T(dy));  dx = dh + LN1^T(Attn^T(dh))
 * Workspace: tp_workspace_size(TP_OP_LAYER_BWD, dims) bytes. */
tp_status tp_layer_bwd(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* params,
                       const tp_layer_acts* acts, const tp_bf16* dy, tp_bf16* dx,
                       const tp_layer_grads* grads, void* ws, size_t ws_bytes, tp_stream stream);

/* tp_layer_bwd_notify: tp_layer_bwd (same arguments and results, bit for bit),
 * for data-parallel training, where each replica's parameter gradients are
 * all-reduced over the replicas ("3D decomposition in practice" and "What
 * actually limits throughput in production": that reduction runs off the
 * critical path, beside the rest of the backward pass).  Each non-NULL
 * member of *ready is a cudaEvent_t (created by the caller on the current
 * device) that is recorded on `stream` as soon as the kernels writing a
 * group of gradients have been enqueued:
 *   mlp   dw1, db1, dw2, db2, dln2_g, dln2_b   (first: the MLP backward runs first)
 *   attn  dwqkv, dbqkv, dwout
 *   ln1   dln1_g, dln1_b, dbout               (last: LN1's backward also sums dbout)
 * A stream that waits on an event may reduce that group while the later
 * kernels of the backward still run.  ready may be NULL (then this is
 * tp_layer_bwd). */
typedef struct {
  void* mlp;    /* cudaEvent_t or NULL */
  void* attn;   /* cudaEvent_t or NULL */
  void* ln1;    /* cudaEvent_t or NULL */
} tp_grad_ready;

tp_status tp_layer_bwd_notify(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* params,
                              const tp_layer_acts* acts, const tp_bf16* dy, tp_bf16* dx,
                              const tp_layer_grads* grads, const tp_grad_ready* ready, void* ws,
                              size_t ws_bytes, tp_stream stream);

/* ------------------------------------------------------------------ activation recomputation
 * "What actually limits throughput in production", the activation memory vs.
 * recomputation trade-off: instead of keeping the layer's activations from
 * the forward to the backward pass, keep only the layer input x and compute
 * them again at the start of the backward pass.
 *
 * tp_layer_fwd_nosave: the pre-LN forward (same result as tp_layer_fwd, bit
 *   for bit) with every intermediate in the workspace; nothing outlives the
 *   call but y.  Workspace: tp_workspace_size(TP_OP_LAYER_FWD_NOSAVE, dims),
 *   about T*(10D + 4F) bytes + the fp16 copy of Wqkv; callers running many
 *   layers can share one workspace between them.
 * tp_layer_bwd_recompute: recomputes the activations of tp_layer_fwd from x
 *   and params into the workspace, then runs tp_layer_bwd on them.  The
 *   recomputed forward leaves out the MLP's second product (y is not needed
 *   for any gradient): 2*T*D*F + 8*T*D^2 + the causal core's forward FLOPs on
 *   top of the backward's.  dx and *grads equal tp_layer_bwd's bit for bit
 *   (same kernels on the same inputs; the library is deterministic).
 *   Workspace: tp_workspace_size(TP_OP_LAYER_BWD_RECOMPUTE, dims) bytes.
 * Arguments, layouts and errors as tp_layer_fwd / tp_layer_bwd. */
tp_status tp_layer_fwd_nosave(const tp_dims* dims, const tp_bf16* x,
                              const tp_layer_params* params, tp_bf16* y, void* ws,
                              size_t ws_bytes, tp_stream stream);
tp_status tp_layer_bwd_recompute(const tp_dims* dims, const tp_bf16* x,
                                 const tp_layer_params* params, const tp_bf16* dy, tp_bf16* dx,
                                 const tp_layer_grads* grads, void* ws, size_t ws_bytes,
                                 tp_stream stream);

/* ------------------------------------------------------------------ post-LN layer
 * The other placement in "The layernorm placement the paper flags as
 * critical": LayerNorm after each residual addition (the original
 * transformer's, the BERT ablation's other arm):
 *   z1 = x + Attn(x);  h = LN1(z1);  z2 = h + MLP(h);  y = LN2(z2)
 * Same parameters (tp_layer_params) and gradients (tp_layer_grads) as the
 * pre-LN layer; the attention sublayer reads x itself. */
typedef struct {
  tp_bf16* z1;            /* x + attention output [T][D] (LN1 input) */
  float *mean1, *rstd1;   /* [T] */
  tp_f16* qkv;            /* [t][T][3Dt], fp16 */
  tp_bf16* o;             /* [t][T][Dt] */
  float* lse;             /* [B][H][S] */
  tp_bf16* h;             /* LN1(z1) [T][D] */
  tp_bf16* z2;            /* h + MLP output [T][D] (LN2 input) */
  float *mean2, *rstd2;   /* [T] */
  tp_bf16* a;             /* MLP pre-activation [t][T][Ft] */
  tp_bf16* hact;          /* MLP activation [t][T][Ft] */
} tp_postln_acts;

/* tp_postln_layer_fwd: x [T][D] -> y [T][D], filling *acts.
 * Workspace: tp_workspace_size(TP_OP_POSTLN_FWD, dims) bytes. */
tp_status tp_postln_layer_fwd(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* params,
                              const tp_postln_acts* acts, tp_bf16* y, void* ws, size_t ws_bytes,
                              tp_stream stream);

/* tp_postln_layer_bwd: dy -> dx and *grads:
 *   dz2 = LN2^T(dy);  dh = dz2 + MLP^T(dz2);  dz1 = LN1^T(dh);  dx = dz1 + Attn^T(dz1)
 * Workspace: tp_workspace_size(TP_OP_POSTLN_BWD, dims) bytes. */
tp_status tp_postln_layer_bwd(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* params,
                              const tp_postln_acts* acts, const tp_bf16* dy, tp_bf16* dx,
                              const tp_layer_grads* grads, void* ws, size_t ws_bytes,
                              tp_stream stream);

/* ------------------------------------------------------------------ LayerNorm
 * The pre-LN building block on its own ("The layernorm placement the paper
 * flags as critical"), exposed for tests and for callers composing layers.
 *   tp_layernorm_fwd: y = (x - mean) * rstd * gamma + beta per row of x [rows][D];
 *                     mean, rstd fp32 [rows].  No workspace.
 *   tp_layernorm_bwd: dx = rstd (g - mean(g) - xhat mean(g xhat)) (+ dres),
 *                     g = dy * gamma; dgamma = sum_rows dy*xhat, dbeta = sum_rows dy.
 *                     dres, dgamma, dbeta may be NULL.
 *                     Workspace: tp_layernorm_bwd_workspace_size(rows, D). */
tp_status tp_layernorm_fwd(const tp_bf16* x, const tp_bf16* gamma, const tp_bf16* beta, int rows,
                           int D, float eps, tp_bf16* y, float* mean, float* rstd, tp_stream stream);
/* tp_layernorm_fwd_f16: tp_layernorm_fwd with an fp16 output y, for a LayerNorm
 * that feeds the attention sublayer's fp16 products (tp_attn_fwd_rank's x16);
 * values beyond the fp16 range set device error 0x301. */
tp_status tp_layernorm_fwd_f16(const tp_bf16* x, const tp_bf16* gamma, const tp_bf16* beta,
                               int rows, int D, float eps, tp_f16* y, float* mean, float* rstd,
                               tp_stream stream);
size_t tp_layernorm_bwd_workspace_size(int rows, int D);
tp_status tp_layernorm_bwd(const tp_bf16* dy, const tp_bf16* x, const tp_bf16* gamma,
                           const float* mean, const float* rstd, const tp_bf16* dres, int rows,
                           int D, tp_bf16* dx, tp_bf16* dgamma, tp_bf16* dbeta, void* ws,
                           size_t ws_bytes, tp_stream stream);

/* tp_layernorm_bwd_noalloc: the same computation as tp_layernorm_bwd, for
 * callers that cannot allocate device memory where they run it (allocator or
 * memory-pool callbacks, runtimes with a fixed memory budget, hot paths where
 * cudaMalloc is forbidden).  The pages have no counterpart to it: it exists
 * for those callers only.  It takes no workspace and allocates nothing; its
 * scratch (the dgamma/dbeta partial sums) is a 4 MiB device array inside the
 * library that every GPU loading the library holds until exit.  All calls on
 * a device share that array: calls whose kernels may overlap on the GPU race
 * and must be serialised by the caller.  The first call on each device looks
 * up the array's device address; make it outside stream capture.  D up to
 * 8192 (wider rows: TP_ERR_UNSUPPORTED); row count unlimited.  dx is
 * identical to tp_layernorm_bwd's; dgamma/dbeta are too while 2 * D * (row
 * blocks, 2 per SM) floats fit the array (D up to 1771 on a 148-SM GPU);
 * wider rows use fewer blocks, which groups the fp32 sums differently
 * (still deterministic). */
tp_status tp_layernorm_bwd_noalloc(const tp_bf16* dy, const tp_bf16* x, const tp_bf16* gamma,
                                   const float* mean, const float* rstd, const tp_bf16* dres,
                                   int rows, int D, tp_bf16* dx, tp_bf16* dgamma, tp_bf16* dbeta,
                                   tp_stream stream);

/* ------------------------------------------------------------------ one shard per GPU
 * The pages' own deployment ("One Idea, Two Insertions" on the explainer;
 * "How transformer layers actually decompose" and "Why TP must stay within a
 * node" on the blog): GPU i of a t-GPU group holds shard i of every weight and
 * the shards meet in one all-reduce per sublayer per direction.  Each call
 * below runs one shard between two exchange points on the calling GPU and
 * writes that shard's PARTIAL of the exchanged tensor, fp32 [T][D], without
 * bias.  The caller sums the t partials (an all-reduce among the ranks, or
 * reads of the peers' buffers) and finishes with tp_rowpar_finish, which adds
 * the row-parallel product's bias once and the residual and rounds once.
 *
 * Every pointer is shard-local (what GPU i holds): W1_i [D][Ft], b1_i [Ft],
 * W2_i [Ft][D], Wqkv_i [D][3Dt] = [Wq_i | Wk_i | Wv_i], bqkv_i [3Dt],
 * Wout_i [Dt][D]; activations of the shard: A_i, H_i [T][Ft], qkv_i [T][3Dt]
 * (fp16), O_i [T][Dt], lse_i [B][H/t][S].  x, dy, the full-width biases b2,
 * bout and the residuals are replicated on every rank.  dims->t is the
 * tensor-parallel degree (the number of ranks); dims describes the WHOLE
 * layer (hidden, ffn, heads), from which the shard widths Ft = F/t,
 * Dt = D/t and the local head count H/t follow.  Workspaces:
 * tp_rank_workspace_size.  Errors and streams as for the other entry points. */
typedef enum {
  TP_RANK_MLP_FWD = 0,
  TP_RANK_MLP_BWD = 1,
  TP_RANK_ATTN_FWD = 2,
  TP_RANK_ATTN_BWD = 3
} tp_rank_op;

/* Bytes of device workspace rank-local operation `op` needs (0 if none or invalid dims). */
size_t tp_rank_workspace_size(int op, const tp_dims* dims);

/* tp_mlp_fwd_rank: a_i = x W1_i + b1_i, h_i = GeLU(a_i) [T][Ft] (saved for the
 * backward); partial = h_i W2_i, fp32 [T][D].  b1_i may be NULL.  No workspace.
 * Finish: y = tp_rowpar_finish(sum of the t partials, b2, resid). */
tp_status tp_mlp_fwd_rank(const tp_dims* dims, const tp_bf16* x, const tp_bf16* w1_i,
                          const tp_bf16* b1_i, const tp_bf16* w2_i, tp_bf16* a_i, tp_bf16* h_i,
                          float* partial, tp_stream stream);

/* tp_mlp_bwd_rank, for the upstream gradient dy [T][D] (replicated):
 *   dA_i = (dy W2_i^T) * GeLU'(a_i);  dw2_i = h_i^T dy [Ft][D];  dw1_i = x^T dA_i [D][Ft];
 *   db1_i = column sums of dA_i [Ft];  db2 = column sums of dy [D] (the same on
 *   every rank; NULL to skip);  partial = dA_i W1_i^T, fp32 [T][D].
 * Finish: dx = tp_rowpar_finish(sum of the t partials, NULL, dres). */
tp_status tp_mlp_bwd_rank(const tp_dims* dims, const tp_bf16* x, const tp_bf16* w1_i,
                          const tp_bf16* w2_i, const tp_bf16* a_i, const tp_bf16* h_i,
                          const tp_bf16* dy, tp_bf16* dw1_i, tp_bf16* dw2_i, tp_bf16* db1_i,
                          tp_bf16* db2, float* partial, void* ws, size_t ws_bytes,
                          tp_stream stream);

/* tp_attn_fwd_rank: the sublayer input as bf16 x or, when the caller already
 * holds it in fp16 (a LayerNorm with fp16 output, tp_layernorm_fwd_f16), as
 * x16; exactly one of the two is non-NULL.  Inside, the products run on fp16
 * operands as in tp_attn_fwd.
 *   qkv_i = x Wqkv_i + bqkv_i [T][3Dt] (fp16; columns [0,Dt) q, [Dt,2Dt) k,
 *   [2Dt,3Dt) v, local head j at j*dh);  per local head: O = softmax(q k^T /
 *   sqrt(dh) + mask) v (fp32 softmax), o_i [T][Dt], lse_i [B][H/t][S];
 *   partial = o_i Wout_i, fp32 [T][D].  bqkv_i may be NULL.
 * Finish: y = tp_rowpar_finish(sum of the t partials, bout, resid). */
tp_status tp_attn_fwd_rank(const tp_dims* dims, const tp_bf16* x, const tp_f16* x16,
                           const tp_bf16* wqkv_i, const tp_bf16* bqkv_i, const tp_bf16* wout_i,
                           tp_f16* qkv_i, tp_bf16* o_i, float* lse_i, float* partial, void* ws,
                           size_t ws_bytes, tp_stream stream);

/* tp_attn_bwd_rank, for dy [T][D] (replicated); x or x16 as in the forward:
 *   dO_i = dy Wout_i^T;  dwout_i = o_i^T dy [Dt][D];  the attention backward of
 *   the local heads (P recomputed from lse_i) gives dqkv_i;  dwqkv_i = x^T dqkv_i
 *   [D][3Dt];  dbqkv_i = column sums of dqkv_i [3Dt];  dbout = column sums of
 *   dy [D] (NULL to skip);  partial = dqkv_i Wqkv_i^T, fp32 [T][D].
 * Finish: dx = tp_rowpar_finish(sum of the t partials, NULL, dres). */
tp_status tp_attn_bwd_rank(const tp_dims* dims, const tp_bf16* x, const tp_f16* x16,
                           const tp_bf16* wqkv_i, const tp_bf16* wout_i, const tp_f16* qkv_i,
                           const tp_bf16* o_i, const float* lse_i, const tp_bf16* dy,
                           tp_bf16* dwqkv_i, tp_bf16* dbqkv_i, tp_bf16* dwout_i, tp_bf16* dbout,
                           float* partial, void* ws, size_t ws_bytes, tp_stream stream);

/* tp_rowpar_finish: out = bf16( parts[0] + parts[1] + ... + parts[nparts-1]
 * + bias + resid ), summed in fp32 in that order and rounded once; out32, when
 * not NULL, receives the same values in fp32.  parts is a HOST array of
 * nparts (1..8) device pointers to fp32 [rows][cols] buffers: one buffer that
 * an all-reduce has already summed, or the t ranks' partials themselves (for
 * example peers' buffers reachable through peer access, read with plain
 * loads).  bias [cols] and resid [rows][cols] may be NULL.  cols % 8 == 0. */
tp_status tp_rowpar_finish(const float* const* parts, int nparts, const tp_bf16* bias,
                           const tp_bf16* resid, int rows, int cols, tp_bf16* out, float* out32,
                           tp_stream stream);

/* ------------------------------------------------------------------ failure-detection self-test
 * Not an operation of the pages: a check of the library's bounded device
 * waits.  tp_selftest_wait_timeout enqueues one small kernel whose thread
 * waits on a barrier that nothing completes, through the same bounded wait
 * every kernel here uses, with limit limit_ns (1 ms to 10 s); when the limit
 * expires it records code 0x0F1 in the device error word and returns.  A
 * following tp_check_error then reports TP_ERR_TIMEOUT with *code == 0x0F1 and
 * clears the word.  Nothing faults or hangs; the context stays usable.
 * INVALID_ARG for a limit outside that range. */
tp_status tp_selftest_wait_timeout(unsigned long long limit_ns, tp_stream stream);

/* ------------------------------------------------------------------ launch trace
 * Measurement support (the pages describe no tracing; this exists so that a
 * bench can time individual kernels inside a longer step on their own stream).
 * tp_trace_begin: from now on, for the i-th kernel the library enqueues
 * (i < capacity), record events[2i] on the launch stream just before it and
 * events[2i+1] just after it, store its class in kinds[i] (0 GEMM, 1 attention
 * forward, 2 attention-backward prep, 3 attention dK/dV, 4 attention dQ,
 * 5 LayerNorm forward, 6 LayerNorm backward, 7 LayerNorm parameter reduce,
 * 8 column sum, 9 layout copy, 10 bf16-to-fp16 conversion, 11 row-parallel finish) and, if
 * flops != NULL, its algorithmic FLOP
 * count in flops[i] (0 for non-contraction kernels).  events are cudaEvent_t
 * handles created by the caller on the current device; arrays are host memory
 * owned by the caller and must stay valid until tp_trace_end.  capacity 0
 * closes the trace.  INVALID_ARG on negative capacity or NULL arrays.
 * tp_trace_end: closes the trace and returns the number of launches seen
 * since tp_trace_begin (which may exceed capacity). */
tp_status tp_trace_begin(void* const* events, int* kinds, double* flops, int capacity);
int tp_trace_end(void);

#ifdef __cplusplus
}
#endif

#endif /* TP_LAYER_H */
