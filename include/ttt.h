/*
 * ttt.h — C ABI of the TTT-E2E inner-loop library (B200, sm_100a).
 *
 * The library runs End-to-End Test-Time Training for long context: a
 * sliding-window-attention Transformer whose MLPs in the last quarter of the
 * blocks ("TTT blocks") are updated at inference by mini-batch gradient descent
 * on next-token cross-entropy. Sources:
 *   - b-lab.team summary of the TTT-E2E paper, "Test-Time Training (Inner
 *     Loop)": loss l_t(W) = CE(f(x_{t-1}; W), x_t) and the mini-batch update
 *     W_i = W_{i-1} - eta * (1/b) * sum_{k in chunk i} grad l_k(W_{i-1});
 *     "Implementation Details for TTT": only MLPs of the last 1/4 of the blocks
 *     update, a static second MLP follows, decode updates after a full
 *     mini-batch of generated tokens.
 *   - "TTT-E2E: Learning a Long Context into Weights" (technical review):
 *     §5 eq. (9) and the sliding window k >= b; §7 Algorithm 1 (causal prefill
 *     with adaptation) and Algorithm 3 (generation with periodic adaptation).
 *
 * Conventions for every entry point:
 *   - Return value: TTT_OK (0) or a negative TTT_ERR_* code. No exceptions
 *     cross the boundary. ttt_last_error() returns a handle-owned message.
 *   - After a CUDA or device-side error the handle is poisoned: later calls
 *     return TTT_ERR_POISONED; only ttt_destroy remains valid.
 *   - Calls are synchronous with respect to the host: they enqueue work on
 *     cfg.cuda_stream and return after the outputs are written.
 *   - Buffers are caller-owned. ptr_kind tells whether a pointer is host
 *     (TTT_PTR_HOST, pageable or pinned) or device (TTT_PTR_DEVICE) memory.
 *   - Not thread-safe per handle; distinct handles are independent.
 */
#ifndef TTT_H
#define TTT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = -1,  /* bad config, size, pointer or token id */
  TTT_ERR_OOM = -2,          /* device allocation failed */
  TTT_ERR_CUDA = -3,         /* a CUDA call failed; handle poisoned */
  TTT_ERR_TIMEOUT = -4,      /* a bounded device wait expired; handle poisoned */
  TTT_ERR_STREAM = -5,       /* stream continuity: first id != pending token, or chunk pending */
  TTT_ERR_POISONED = -6,     /* handle unusable after an earlier device error */
  TTT_ERR_UNSUPPORTED = -7   /* shape the kernels do not support */
};

enum { TTT_FP32 = 0, TTT_BF16 = 1 };

/* Inner loss that drives the fast-weight update (ttt_config.inner_loss).
 *   TTT_LOSS_E2E: the next-token cross-entropy at the model's output, back-propagated
 *     into every adaptive MLP (summary, "Test-Time Training (Inner Loop)"; technical
 *     review §5 eq. (9)).
 *   TTT_LOSS_KVB: the layer-wise key-value-binding variant (technical review §8,
 *     eq. (10); summary, "Alternative Derivation (Connection to TTT-KVB)"): each
 *     adaptive block fits its MLP g(k; W) = W2t gelu(W1t k) from k = theta_K x to
 *     v = theta_V x, x the MLP's own normalised input, minimising
 *     (1/b) sum_t ||g(theta_K x_t; W) - theta_V x_t||^2 over the chunk with respect
 *     to its own W only. theta_K, theta_V are frozen [d][d] matrices of the block.
 *     The recorded per-token losses stay the next-token losses under W_{i-1}. */
enum { TTT_LOSS_E2E = 0, TTT_LOSS_KVB = 1 };
enum { TTT_PTR_HOST = 0, TTT_PTR_DEVICE = 1 };

typedef struct ttt_handle ttt_handle;

/* Model and inner-loop hyper-parameters. Notation: V vocab, d width, L layers,
 * L_t adaptive (last) layers, H heads (head dim d/H), k window, b mini-batch.
 * n_ttt = L_t may be 0: no block adapts, and the handle is the plain SWA
 * Transformer (full causal attention when window_k >= T), whose prefill records
 * the per-position losses only. It is the comparator the summary's speed claim
 * is made against (TTT-E2E vs full attention at 128K, "Results"). */
typedef struct {
  int32_t vocab, d, n_layers, n_heads, n_ttt;
  int32_t mlp_hidden;     /* frozen blocks' MLP hidden width h */
  int32_t ttt_hidden;     /* h_t: adaptive MLP hidden width (fast weights W1t [h_t][d], W2t [d][h_t]) */
  int32_t static_hidden;  /* h_s: static second MLP hidden width in adaptive blocks */
  int32_t window_k;       /* sliding-window length k (>= minibatch_b) */
  int32_t minibatch_b;    /* inner mini-batch b */
  int32_t batch;          /* B independent sequences, each with its own fast weights */
  float eta;              /* inner step size */
  float rms_eps;          /* RMSNorm epsilon inside the root */
  float rope_base;        /* RoPE base */
  int32_t dtype;          /* TTT_FP32 (fp32 everywhere) or TTT_BF16 (bf16 operands, fp32 accumulation and master fast weights) */
  int32_t max_segment;    /* positions per sequence processed per frozen-phase segment (0 = default 32768; rounded to b) */
  int32_t inner_loss;     /* TTT_LOSS_E2E (default, 0) or TTT_LOSS_KVB */
  void* cuda_stream;      /* cudaStream_t to run on (NULL = legacy default stream) */
} ttt_config;

/* Weights: an array of n_tensors pointers in this fixed order (each tensor
 * row-major, matrices stored [out][in] so that y = x W^T):
 *   E [V][d] (embedding, tied LM head), final_norm [d],
 *   then for every layer l = 0..L-1:
 *     attn_norm [d], Wq [d][d], Wk [d][d], Wv [d][d], Wo [d][d],
 *     frozen layer (l < L - L_t): mlp_norm [d], W1 [h][d], W2 [d][h]
 *     TTT layer    (l >= L - L_t): ttt_norm [d], W1t [h_t][d], W2t [d][h_t],
 *                                  static_norm [d], W1s [h_s][d], W2s [d][h_s],
 *                                  and with inner_loss == TTT_LOSS_KVB also
 *                                  theta_K [d][d], theta_V [d][d]
 * values_dtype: element type of the given arrays (TTT_FP32 float32, or TTT_BF16 raw bf16 bits);
 * norm gains are always float32. The library copies everything; the caller keeps its buffers. */
typedef struct {
  const void* const* tensors;
  int32_t n_tensors;
  int32_t values_dtype;
  int32_t ptr_kind;
} ttt_weights;

/* Number of tensors ttt_weights must hold for cfg. */
int32_t ttt_num_weight_tensors(const ttt_config* cfg);

/* Validate cfg (k >= b, d % H == 0, widths multiples of 8, ...), allocate
 * device state (frozen weights, B copies of the fast weights W_init as fp32
 * master + bf16 shadow, window caches of roundup(k + b, 128) positions per
 * layer and sequence, workspace) and copy the weights (review §7, Algorithm 1:
 * every sequence starts from a fresh copy of W_init). *out receives the handle
 * (NULL on failure). On failure nothing is leaked. */
int ttt_create(const ttt_config* cfg, const ttt_weights* w, ttt_handle** out);

/* Algorithm 1 over T positions of each of the B sequences.
 * tokens [B][T+1] int32 (x_0..x_T per sequence, row stride T+1): positions 0..T-1
 * are processed and out_losses[b][t-1] = l_t = -log p(x_t | x_<t) for t = 1..T,
 * every loss of chunk i scored with W_{i-1} before the update (review §5 and
 * Algorithm 1). Chunks are the global grid [(i-1)b, ib) of positions since
 * creation/reset; a chunk updates W only when complete; a trailing partial
 * chunk stays pending (decode completes it). x_T becomes the pending input.
 * A continuing call must start with the pending id (else TTT_ERR_STREAM) and
 * may not start while a partial chunk is pending (TTT_ERR_STREAM).
 * Token ids must lie in [0, V) (else TTT_ERR_INVALID_ARG, checked on the device). */
int ttt_prefill(ttt_handle* h, const int32_t* tokens, int64_t T, float* out_losses, int32_t ptr_kind);

/* Algorithm 3: generate n tokens per sequence. Each step feeds the pending
 * token, takes the argmax of the logits (lowest id on ties) — or, when forced
 * is non-NULL, the id forced[b][t] — writes it to out_tokens[b][t] and
 * -log p(chosen) to out_losses[b][t] (may be NULL). When a chunk of b
 * positions completes, its inner loss (the chunk's mean next-token loss, or
 * with TTT_LOSS_KVB each adaptive block's binding loss) is differentiated and
 * W updated (summary, "Decoding Multiple Tokens"). forced/out_* use ptr_kind. */
int ttt_decode(ttt_handle* h, int64_t n, const int32_t* forced, int32_t* out_tokens, float* out_losses,
               int32_t ptr_kind);

/* Copy the fp32 fast weights of sequence seq, adaptive block j (0 = first TTT block):
 * w1 [h_t][d] and w2 [d][h_t] (either may be NULL). These are the adapted W that
 * Algorithm 1 of the technical review (§7) returns beside the attention state: W_init
 * after every completed chunk's update so far. ptr_kind: host or device buffers. */
int ttt_get_weights(ttt_handle* h, int32_t seq, int32_t ttt_block, float* w1, float* w2, int32_t ptr_kind);

/* Fast weights <- W_init, window caches and pending state cleared (review §7,
 * Algorithm 2: adapted state is discarded between documents). */
int ttt_reset(ttt_handle* h);

/* Positions processed so far (per sequence). */
int64_t ttt_position(const ttt_handle* h);

/* Device bytes held by the handle (the per-session budget of review eq. (13)). */
int64_t ttt_device_bytes(const ttt_handle* h);

/* Kernel launches issued by the most recent prefill or decode call. */
int64_t ttt_last_launch_count(const ttt_handle* h);

/* Kernel-class timing. When enabled, CUDA events are recorded on the handle's
 * stream around every launch of these classes, and the algorithmic work of each
 * launch is counted: 0 frozen-phase GEMMs, 1 adaptive-phase GEMMs, 2 attention
 * forward, 3 attention backward. FLOPs: 2*M*N*K per GEMM; attention 4*hd*H per
 * query-key pair of the window forward (review eq. (1) counts the pairs), and
 * 2*hd*H*(2 window pairs + 2 current-chunk pairs) backward (no recompute counted). Bytes: operands read
 * once plus the output written once. ttt_profile(h, 1) clears the counters.
 * ttt_profile_read fills up to n_classes entries (any pointer may be NULL) and
 * returns the number of classes. Accumulates over calls until cleared. */
int ttt_profile(ttt_handle* h, int32_t enable);
int ttt_profile_read(const ttt_handle* h, int32_t n_classes, double* ms, int64_t* launches, double* flops,
                     double* bytes);

void ttt_destroy(ttt_handle* h);

const char* ttt_last_error(const ttt_handle* h);

/* Library build string. */
const char* ttt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H */
