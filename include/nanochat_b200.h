/*
 * nanochat_b200.h -- C ABI of the B200 (sm_100a) forward+backward pretraining
 * step of the nanochat-style dense decoder.
 *
 * The model is the one listed in the architecture section of the nanochat
 * announcement (vpshk.cn, "Andrej Karpathy open-sources nanochat"): a dense,
 * Llama-like decoder with rotary position embeddings only, QK-norm, untied
 * embedding and unembedding, a normalised token embedding, a relu^2 MLP,
 * parameter-free RMSNorm, bias-free linears, multi-query attention and a
 * tanh logit softcap.  The loss is the mean next-token cross-entropy over all
 * B*T positions, and the step returns the gradient of that mean with respect
 * to every weight.  Readings of points the pages leave open (RMSNorm eps,
 * final norm, RoPE pairing and frequencies, attention scale, causal mask) are
 * fixed here and stated next to the declarations they affect.
 *
 * Conventions for every entry point:
 *   - Pointers named d_* or documented as "device" are device memory owned by
 *     the caller.  The library never frees them and never keeps them after the
 *     call returns (it only enqueues work that reads or writes them).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work; they do not synchronise, except
 *     nc_check and nc_forward_backward_host (see there).
 *   - Return values are NC_OK (0) or a negative NC_ERR_* code describing
 *     argument validation or launch failure.  Errors found on the device
 *     (token id out of range, a bounded wait that expired) are recorded in a
 *     device status word owned by the model and reported by nc_check.
 *   - All matrices are row-major.  A linear layer is y = x W^T with W stored
 *     [out, in].
 */
#ifndef NANOCHAT_B200_H
#define NANOCHAT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define NC_OK                       0
#define NC_ERR_INVALID_ARG         -1  /* null pointer, non-positive size, bad index,
                                          misaligned buffer, or not the model's device */
#define NC_ERR_UNSUPPORTED_SHAPE   -2  /* config outside what the kernels implement      */
#define NC_ERR_WORKSPACE_TOO_SMALL -3  /* ws_bytes < nc_workspace_bytes(model, B, T)      */
#define NC_ERR_CUDA                -4  /* a CUDA runtime call or kernel launch failed    */
#define NC_ERR_BAD_TOKEN           -5  /* device: a token or target id outside [0, V)    */
#define NC_ERR_DEVICE_TIMEOUT      -6  /* device: a bounded wait in a kernel gave up     */
#define NC_ERR_NO_DEVICE           -7  /* no sm_100 device current when the model was made */

/* Parameter-free RMSNorm epsilon: y = x / sqrt(mean(x^2) + NC_RMS_EPS).  The
 * pages give no value; 1e-6 is used everywhere (token-embedding norm, the two
 * pre-norms of every block, QK-norm, final norm). */
#define NC_RMS_EPS 1e-6f

/* Model shape.  d_model = n_head*head_dim is not required.  MLP hidden width
 * is mlp_mult*d_model.  Supported: d_model % 64 == 0, head_dim in
 * {16, 32, 64, 128}, n_head % n_kv_head == 0, vocab % 64 == 0, softcap > 0,
 * rope_base > 1.  RoPE rotates the pairs (j, j + head_dim/2) of every q and
 * k head by pos * rope_base^(-2j/head_dim), positions 0..T-1 in each row. */
typedef struct {
    int vocab, d_model, n_layer, n_head, n_kv_head, head_dim, mlp_mult;
    float softcap, rope_base;
} nc_config;

/* Arithmetic of the step.
 * NC_PREC_BF16: bf16 weights, bf16 GEMM/attention operands on the tcgen05
 *   tensor cores with fp32 accumulation; fp32 residual stream, norm
 *   statistics, softmax and loss.
 * NC_PREC_FP32_DEBUG: fp32 weights and activations everywhere, plain fp32
 *   FMA kernels (no tensor cores, no TF32). */
typedef enum { NC_PREC_BF16 = 0, NC_PREC_FP32_DEBUG = 1 } nc_precision;

typedef struct nc_model nc_model; /* opaque */

/* Validates cfg and creates a model bound to the current CUDA device.  Host
 * state plus one small device status word (allocated here, freed by
 * nc_model_destroy).  *out is set to NULL on error.  That device must be the
 * current one whenever a step, logits or debug call is made on the model:
 * those calls return NC_ERR_INVALID_ARG, launching nothing, when another
 * device is current (its kernels would otherwise reach the buffers as peer
 * memory). */
int nc_model_create(const nc_config* cfg, nc_precision prec, nc_model** out);
void nc_model_destroy(nc_model* m);

/* Number of parameter elements (= elements of the flat weight and gradient
 * buffers). */
int64_t nc_num_params(const nc_model* m);

/* Flat parameter layout, entry i in [0, 2 + 6*n_layer): name, element offset,
 * rows, cols.  Order: "wte" [V,d]; per layer i "h.i.wq" [H*hd,d],
 * "h.i.wk" [nkv*hd,d], "h.i.wv" [nkv*hd,d], "h.i.wo" [d,H*hd],
 * "h.i.wfc" [F,d], "h.i.wproj" [d,F]; then "wlm" [V,d].  *name points to
 * library-owned storage valid for the model's lifetime. */
int nc_param_layout(const nc_model* m, int i, const char** name, int64_t* offset,
                    int* rows, int* cols);

/* Bytes of device workspace nc_forward_backward / nc_forward_logits need for
 * batch B and sequence length T.  Returns 0 for invalid B, T. */
size_t nc_workspace_bytes(const nc_model* m, int B, int T);

/* One forward+backward step (the hot path).
 *   tokens, targets: device int32 [B, T], row-major contiguous.  targets are
 *     the next-token ids (tokens shifted by one in the caller's stream).
 *   weights: device, nc_num_params elements, bf16 (NC_PREC_BF16) or fp32
 *     (NC_PREC_FP32_DEBUG), in the nc_param_layout order.
 *   grads: device fp32, nc_num_params elements; OVERWRITTEN with the gradient
 *     of the mean loss (not accumulated).
 *   loss: device fp32 scalar; receives mean_{b,t} [logsumexp(z) - z[target]]
 *     with z = softcap * tanh(logits / softcap).
 *   workspace: device, at least nc_workspace_bytes(m, B, T) bytes, 256-byte
 *     aligned; its contents on entry are ignored.
 * The full [B*T, V] logit tensor is never written to memory.  Results are
 * bitwise reproducible for a given model, inputs and workspace size.
 * Streams: the step is enqueued on `stream` (NULL = the legacy default
 * stream); the weight-gradient GEMMs of the backward pass may run on a second
 * stream owned by the model, forked from and joined back into `stream` with
 * events, so every write of the call is ordered before work the caller
 * enqueues on `stream` afterwards.  A model runs one call at a time: calls on
 * the same model from several host threads, or interleaved on several
 * streams, must be serialised by the caller. */
int nc_forward_backward(nc_model* m, const int32_t* tokens, const int32_t* targets,
                        int B, int T, const void* weights, float* grads, float* loss,
                        void* workspace, size_t ws_bytes, void* stream);

/* Same step with the per-step inputs and the result in HOST memory:
 * h_tokens / h_targets are host int32 [B, T] (pinned memory gives an
 * asynchronous copy), h_loss a host float.  The ids are copied into the
 * workspace, the step is enqueued on `stream`, the loss is copied back, and
 * the call synchronises `stream` before returning.  Weights, grads and the
 * workspace are device memory as for nc_forward_backward. */
int nc_forward_backward_host(nc_model* m, const int32_t* h_tokens, const int32_t* h_targets,
                             int B, int T, const void* weights, float* grads, float* h_loss,
                             void* workspace, size_t ws_bytes, void* stream);

/* Forward pass only; writes the softcapped logits z [B, T, V] (bf16 for
 * NC_PREC_BF16, fp32 for NC_PREC_FP32_DEBUG) to the device buffer `logits`.
 * This is the only call that materialises the logits of every position.  It
 * needs only nc_inference_workspace_bytes(m, B, T) bytes of workspace (the
 * forward alone); nc_workspace_bytes(m, B, T) is more than enough. */
int nc_forward_logits(nc_model* m, const int32_t* tokens, int B, int T, const void* weights,
                      void* logits, void* workspace, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then returns and clears the device status word:
 * NC_OK, NC_ERR_BAD_TOKEN or NC_ERR_DEVICE_TIMEOUT (or NC_ERR_CUDA if the
 * stream reported an error). */
int nc_check(nc_model* m, void* stream);

/* Static description of a return code. */
const char* nc_status_string(int code);

/* Per-kernel-class timing.  While enabled, every launch made by this model
 * is bracketed by CUDA events on its stream, tagged with the kernel class and
 * the algorithmic work of the call (FLOPs for contractions, HBM bytes for the
 * memory-bound kernels).  nc_profile_enable(m, 1) clears the record and
 * starts; (m, 0) stops.  nc_profile_read synchronises `stream` and writes up
 * to max_rows aggregated rows (one per kernel class seen); returns the number
 * of rows or a negative code.  `kernel` points to static storage. */
typedef struct {
    const char* kernel;
    int64_t launches;  /* kernel launches of this class */
    double ms;         /* summed event time */
    double flops;      /* algorithmic FLOPs */
    double bytes;      /* algorithmic HBM bytes */
} nc_profile_row;
int nc_profile_enable(nc_model* m, int enable);
int nc_profile_read(nc_model* m, void* stream, nc_profile_row* rows, int max_rows);

/* Kernels launched by the library in this process so far. */
int64_t nc_launch_count(void);

/* Gradient buckets for data-parallel averaging, in the order in which the
 * backward of nc_forward_backward finishes them: bucket 0 is the LM head
 * (wlm), bucket 1 + k the six matrices of layer n_layer - 1 - k (adjacent in
 * the flat layout), bucket n_layer + 1 the token embedding (wte).
 *   nc_grad_bucket_count: n_layer + 2, or NC_ERR_INVALID_ARG for a null handle.
 *   nc_grad_bucket: element offset and element count of bucket i in the flat
 *   gradient buffer; NC_ERR_INVALID_ARG for a null argument or i out of range.
 * Host-only: neither call touches the device. */
int nc_grad_bucket_count(const nc_model* m);
int nc_grad_bucket(const nc_model* m, int i, int64_t* offset, int64_t* count);

/* Optional per-bucket completion events, for overlapping a gradient exchange
 * with the backward.  events: n cudaEvent_t handles passed as void*, created
 * and owned by the caller, with n == nc_grad_bucket_count(m); n == 0 (events
 * may be NULL) clears them.  While they are set, nc_forward_backward and
 * nc_forward_backward_host record event i on the step's stream as soon as
 * bucket i of the gradients is final, so another stream can wait on it and
 * reduce that bucket while the backward continues.  The events must stay
 * valid while set.  NC_ERR_INVALID_ARG for a null handle, a wrong n or a null
 * event; nothing is recorded by this call itself. */
int nc_set_grad_events(nc_model* m, void* const* events, int n);

/* Inference with a KV cache (the nanochat pipeline's inference engine with
 * prefill and decode, tianqi.csdn.net pipeline paragraph).  Multi-query
 * attention keeps one K and one V head per K/V group: the cache is
 * [n_layer] x {K, V} x [B, T_max, n_kv_head, head_dim] in the weights' type
 * (K after QK-norm and RoPE), nc_kv_cache_bytes(m, B, T_max) bytes of device
 * memory owned by the caller, passed unchanged from the prefill to every
 * decode step of the same B rows.
 *   nc_inference_workspace_bytes: workspace for nc_prefill with any T <= T_max
 *     and for nc_decode_step (0 for bad sizes).
 *   nc_prefill: the forward over tokens [B, T] (device int32, every row T
 *     long), cache positions 0..T-1 written, softcapped logits of position T-1
 *     of every row into logits [B, V] (weights' type).
 *   nc_decode_step: one new token per row, tokens [B] (device int32), at
 *     position pos (the number of positions already cached, same for every
 *     row; pos < T_max): writes that position's k, v into the cache and the
 *     softcapped logits [B, V] of the new position, attending to 0..pos.
 * Errors as nc_forward_logits, plus NC_ERR_INVALID_ARG for T > T_max or pos
 * outside [0, T_max).  Both only enqueue on `stream`. */
size_t nc_kv_cache_bytes(const nc_model* m, int B, int T_max);
size_t nc_inference_workspace_bytes(const nc_model* m, int B, int T_max);
int nc_prefill(nc_model* m, const int32_t* tokens, int B, int T, const void* weights, void* kv_cache, int T_max,
               void* logits, void* workspace, size_t ws_bytes, void* stream);
int nc_decode_step(nc_model* m, const int32_t* tokens, int B, int pos, const void* weights, void* kv_cache,
                   int T_max, void* logits, void* workspace, size_t ws_bytes, void* stream);

/* LM head strategy of nc_forward_backward (both never hold the full [B*T, V]
 * logit tensor; B*T rows are processed R at a time):
 *   NC_LM_HEAD_FUSED (default on the bf16 path; bf16 only): the logit GEMM's
 *     epilogue applies the softcap z = cap tanh(l/cap) and, because |z| <= cap,
 *     writes u = exp(z - cap) (1 - (z/cap)^2) and per-tile sums of exp(z - cap)
 *     instead of the logits; a row pass forms the loss (cap + log S - z[target])
 *     and folds the one-hot term into u, and the two backward products read u
 *     with a per-row factor 1 / (S B T).  The logits are never written.
 *   NC_LM_HEAD_MATERIALISED (the fp32 debug path's only mode): the softcapped
 *     logits of R rows are written, a cross-entropy pass reads them and writes
 *     their gradient, and the backward products read that.
 * chunk_rows: R (0 = the default: R V elements near 512 MiB fused, 1 GiB
 * materialised).  Changes nc_workspace_bytes.  NC_ERR_INVALID_ARG for an
 * unknown mode, a negative chunk_rows, or FUSED on the fp32 debug path. */
#define NC_LM_HEAD_FUSED 0
#define NC_LM_HEAD_MATERIALISED 1
int nc_set_lm_head(nc_model* m, int mode, int chunk_rows);

/* AdamW update of (ranges of) the flat parameter vector, the optimizer the
 * announcement names beside Muon (vpshk.cn, optimizer paragraph: Muon +
 * AdamW, with a plan to use Adam alone with a learning rate per module).  Muon
 * is not defined on the pages and is not provided.  Textbook AdamW (Adam,
 * Kingma & Ba 2015, with decoupled weight decay, Loshchilov & Hutter 2019);
 * for every element of each group, with t = step (1 for the first update):
 *   m <- b1 m + (1 - b1) g;   v <- b2 v + (1 - b2) g^2
 *   theta <- theta - lr (wd theta + (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps))
 *   weights <- theta in the step's type (bf16 rounded to nearest even, or fp32)
 * groups: n_groups (1..NC_ADAMW_MAX_GROUPS) host descriptors of disjoint
 *   element ranges [offset, offset + count) of the flat layout, each with its
 *   own hyper-parameters (0 <= beta < 1, eps > 0, lr >= 0, weight_decay >= 0).
 * master, grads, m, v: device fp32 [n_params]; weights: device [n_params],
 *   bf16 when weights_bf16 != 0, else fp32.  All five 16-byte aligned; m and v
 *   start at zero before step 1 (the caller clears them).  Elements outside
 *   every group are not touched.
 * One kernel on `stream`.  NC_ERR_INVALID_ARG for a null or misaligned
 * pointer, step < 1, a range outside [0, n_params) or a bad hyper-parameter. */
#define NC_ADAMW_MAX_GROUPS 16
typedef struct {
    int64_t offset, count;
    float lr, beta1, beta2, eps, weight_decay;
} nc_adamw_group;
int nc_adamw_step(const nc_adamw_group* groups, int n_groups, int64_t n_params, int step, float* master,
                  void* weights, int weights_bf16, const float* grads, float* m, float* v, void* stream);

/* Activation recomputation (the llm.c training command's option to
 * recompute activations in the backward, qian.cx llm.c article): with
 * NC_RECOMPUTE_MLP, nc_forward_backward keeps relu(u) and relu(u)^2 of the MLP
 * in one slot shared by all layers and recomputes them from the saved input
 * of the MLP (one extra up-projection GEMM per layer but the last) in the
 * backward, instead of saving them per layer: 2 * 2 * B*T * mlp_mult*d_model
 * bytes per layer less workspace (bf16).  The results are bitwise those of
 * NC_RECOMPUTE_NONE (the same GEMM runs again on the same operands).  Changes
 * nc_workspace_bytes.  NC_ERR_INVALID_ARG for unknown flags. */
#define NC_RECOMPUTE_NONE 0
#define NC_RECOMPUTE_MLP 1
int nc_set_recompute(nc_model* m, int flags);

/* Weight-gradient GEMM that allocates no memory at all.
 *
 * No counterpart in the paper: this is an extra entry point of this library.
 * Some callers cannot call cudaMalloc: frameworks whose caching allocator
 * reserves the device memory up front and owns every later allocation,
 * latency-critical loops where an allocation (which may synchronise the
 * device) is not acceptable, and hosts with a fixed memory budget fixed at
 * start-up.  They can still pass their own inputs and outputs.
 *
 * Computes dw[o, i] (+)= sum_{t < rows} dy[t, o] * x[t, i] -- the gradient of a
 * bias-free linear y = x W^T -- on the tcgen05 tensor cores:
 *   dy: device bf16 [rows, ld_dy] (first n_out columns used)
 *   x:  device bf16 [rows, ld_x]  (first n_in columns used)
 *   dw: device fp32 [n_out, n_in], contiguous; overwritten, or added to when
 *       accumulate != 0
 *   status: device int status word for the bounded waits (may be NULL)
 * dy, x and dw must start on a 16-byte boundary and ld_dy, ld_x must be
 * multiples of 8 (16-byte rows); otherwise the call returns
 * NC_ERR_INVALID_ARG before anything is launched.
 *
 * Split-K partial sums live in one file-scope static device array of
 * NC_WGRAD_NOALLOC_SCRATCH_BYTES; every GPU that loads the library holds it
 * until the process exits.  Results of shape n_out * n_in * 4 * 2 bytes
 * larger than that array (room for two partials) are rejected with
 * NC_ERR_UNSUPPORTED_SHAPE.  Every call shares the array and it keeps the
 * last call's contents; each call overwrites every partial it reads, so
 * nothing has to start at zero.  Calls that overlap on the GPU (other
 * streams, other host threads) race on the array: serialise them.  The first
 * call on a device looks up the array's device address with
 * cudaGetSymbolAddress (with that device current); make that first call
 * before any stream capture. */
#define NC_WGRAD_NOALLOC_SCRATCH_BYTES (64u << 20)
int nc_gemm_wgrad_noalloc(int rows, int n_out, int n_in, const void* dy, int64_t ld_dy, const void* x,
                          int64_t ld_x, float* dw, int accumulate, int* status, void* stream);

/* Test hook for the bounded device wait: launches one kernel that waits on an
 * mbarrier nobody arrives at, with an iteration cap of `max_iters`; when the
 * cap is hit the kernel records NC_ERR_DEVICE_TIMEOUT in the status word and
 * returns (no trap, the context stays usable).  Read the result with
 * nc_check. */
int nc_debug_expired_wait(nc_model* m, int max_iters, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* NANOCHAT_B200_H */
