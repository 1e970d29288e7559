/*
 * mk — one auto-regressive decode step of a decoder-only transformer as ONE
 * persistent CUDA kernel for NVIDIA B200 (sm_100a).
 *
 * The operation is the decode step of ForgeMegakernel (arXiv 2609.12379,
 * abstract): per token, embed -> for every layer [RMSNorm, Q/K/V projection,
 * optional per-head q/k RMSNorm, RoPE, KV-cache append, attention over the
 * cache, output projection + residual, RMSNorm, SwiGLU MLP or top-k MoE +
 * residual] -> final RMSNorm -> LM head.  The abstract names the structural
 * properties the kernel follows: a fine-grained instruction stream per SM and
 * dependency counters in place of grid-wide synchronisation.
 *
 * Conventions of every entry point:
 *   - Plain C types only.  Pointers documented "device" must be device
 *     memory of the current CUDA device; "host" pointers are host memory.
 *   - Return value: MK_OK (0) or a negative mk_status code.  No call aborts
 *     or throws.  mk_status_string() names a code.
 *   - A handle is not thread-safe: calls on one handle must be serialised.
 *
 * Data types: weights and the KV cache are bfloat16 (bit patterns, 2 bytes);
 * activations and logits are float32; token ids, positions and lengths are
 * int32.  All weight matrices are row-major [out][in] (y = W x), every
 * weight/cache pointer 16-byte aligned.
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mk_status {
  MK_OK = 0,
  MK_ERR_INVALID_ARG = -1,    /* NULL pointer, non-positive size, bad enum */
  MK_ERR_UNSUPPORTED = -2,    /* shape, alignment or device not supported */
  MK_ERR_CUDA = -3,           /* a CUDA runtime call failed (allocation, launch) */
  MK_ERR_DEVICE_TIMEOUT = -4, /* a bounded in-kernel wait ran out; the step was abandoned */
  MK_ERR_RANGE = -5           /* seq_lens/positions/tokens out of range (detected on the device) */
} mk_status;

/* Model shape, fixed at creation (all sizes in elements). */
typedef struct mk_model_desc {
  int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn_dim, vocab;
  int32_t n_experts, top_k, expert_ffn_dim; /* n_experts == 0: dense SwiGLU MLP */
  int32_t qk_norm;                          /* 1: per-head RMSNorm of q and k (gain [head_dim]) before RoPE */
  int32_t tied_embeddings;                  /* 1: LM head is the embedding matrix */
  float rms_eps, rope_theta;
  int32_t batch;                            /* sequences decoded together */
  int32_t max_ctx;                          /* KV-cache capacity (positions) per sequence */
  uint64_t wait_timeout_ns;                 /* bound of every in-kernel wait; 0 -> 2 s */
} mk_model_desc;

/* Per-layer weights (device, bf16).  Shapes with H = hidden, D = head_dim:
 *   attn_norm, mlp_norm [H]; q_norm, k_norm [D] (qk_norm only, else NULL)
 *   wq [n_q_heads*D][H]; wk, wv [n_kv_heads*D][H]; wo [H][n_q_heads*D]
 *   dense:  w_gate, w_up [ffn_dim][H]; w_down [H][ffn_dim]; router NULL
 *   MoE:    w_gate, w_up [n_experts][expert_ffn_dim][H] (stacked);
 *           w_down [n_experts][H][expert_ffn_dim]; router [n_experts][H] */
typedef struct mk_layer_weights {
  const void *attn_norm, *wq, *wk, *wv, *q_norm, *k_norm, *wo, *mlp_norm;
  const void *w_gate, *w_up, *w_down, *router;
} mk_layer_weights;

/* Model-global weights (device, bf16): embed [vocab][H], final_norm [H],
 * lm_head [vocab][H] (ignored when tied_embeddings).  layers: HOST array of
 * n_layers entries, read during mk_create only. */
typedef struct mk_weights {
  const void *embed, *final_norm, *lm_head;
  const mk_layer_weights* layers;
} mk_weights;

/* KV cache (device, bf16, caller-owned).
 * Contiguous (block_table == NULL): k and v are each
 *   [n_layers][batch][n_kv_heads][max_ctx][head_dim].
 * Paged (block_table != NULL): k and v are page pools
 *   [n_layers][n_pages][n_kv_heads][page_size][head_dim], and block_table
 *   (device int32 [batch][ceil(max_ctx / page_size)], caller-owned, may be
 *   rewritten between steps) maps page j of a sequence (positions
 *   [j*page_size, (j+1)*page_size)) to a pool page.  page_size must be a
 *   multiple of one attention stage, 32768 / (2*head_dim) positions (128 at
 *   head_dim 128); every page a step reads or writes must be < n_pages
 *   (checked on the device: MK_ERR_RANGE). */
typedef struct mk_kv {
  void *k, *v;
  const int32_t* block_table;
  int32_t page_size, n_pages;
} mk_kv;

typedef struct mk_handle mk_handle;

/*
 * Validate the shape, lower the model into per-SM instruction lists, and
 * allocate the library-owned device state (instruction lists, dependency
 * counters, activation scratch, RoPE cos/sin table) on the current device.
 * Weight and cache pointers are borrowed: they must stay valid until
 * mk_destroy and are never freed by the library.
 * Returns MK_ERR_UNSUPPORTED for shapes the kernel cannot run:
 *   - head_dim not 64 or 128; n_q_heads not 1, 2, 4 or 8 times n_kv_heads;
 *   - batch > 8;
 *   - a GEMV width (hidden, n_q_heads*head_dim, ffn_dim or expert_ffn_dim)
 *     not a multiple of 8;
 *   - batch > 1 or MoE (the tensor-core kernel) with hidden, n_q_heads*head_dim,
 *     ffn_dim or expert_ffn_dim not a multiple of 64;
 *   - MoE with more than 256 experts, top_k > 8, or batch * top_k > 64;
 *   - max_ctx * head_dim above 2^31; misaligned pointers; a device without
 *     cooperative launch or the shared memory the kernel needs.
 * MK_ERR_INVALID_ARG for a malformed description (non-positive sizes, a
 * negative eps, a non-positive rope_theta, top_k outside 1..n_experts).
 */
int mk_create(const mk_model_desc* desc, const mk_weights* weights, const mk_kv* kv, mk_handle** out);

/*
 * One decode step for every sequence, asynchronous on `stream` (a
 * cudaStream_t; NULL = legacy default stream): one kernel launch, no host
 * synchronisation and no allocation.
 *   tokens    device int32[batch]  token id entering the model
 *   positions device int32[batch]  RoPE position of that token (normally seq_lens[b])
 *   seq_lens  device int32[batch]  tokens already cached; the step writes the new K/V
 *                                  row at index seq_lens[b] and attends over
 *                                  seq_lens[b]+1 positions.  The caller advances it.
 *   out_logits device float[batch][vocab]
 * A device-side failure (range error, wait timeout) is reported by
 * mk_get_status; until then later steps return at once without computing.
 */
int mk_decode_step(mk_handle* h, const int32_t* tokens, const int32_t* positions, const int32_t* seq_lens,
                   void* stream, float* out_logits);

/*
 * On-device greedy decoding: n_steps decode steps back to back on `stream`,
 * with no host round trip between them.  Step t runs every sequence b on
 * token x_t[b] at position and cache index seq_lens[b] + t (appending its
 * K/V there), then picks x_{t+1}[b] = argmax of its logits (the largest
 * logit; among equal logits the lowest token id).
 *   tokens     device int32[batch]: x_0, the first step's tokens
 *   seq_lens   device int32[batch]: cached tokens before the first step
 *              (positions equal lengths throughout; both arrays are only read)
 *   out_tokens device int32[n_steps][batch]: x_1 .. x_{n_steps}
 *   out_logits device fp32[batch][vocab] for the last step's logits, or NULL
 * Asynchronous on `stream`; device-side errors (e.g. a length reaching
 * max_ctx, MK_ERR_RANGE) are reported by mk_get_status, which the caller must
 * check after the loop: the return value only covers argument checks and
 * launches.  Once a step fails, the later steps of the call do no work and
 * out_tokens holds -1 for the failing step and every step after it.  Each step
 * is the same kernel as mk_decode_step; the pick folds the LM head's outputs
 * into per-sequence maxima on the device and a one-warp kernel advances the
 * state.
 */
int mk_decode_greedy(mk_handle* h, int n_steps, const int32_t* tokens, const int32_t* seq_lens, void* stream,
                     int32_t* out_tokens, float* out_logits);

/* Synchronise `stream` and return the device-side status of the last steps
 * (MK_OK, MK_ERR_DEVICE_TIMEOUT or MK_ERR_RANGE).  A failure is cleared and
 * the dependency counters are reset, so the handle is usable again. */
int mk_get_status(mk_handle* h, void* stream);

/* Free the library-owned device state.  NULL is accepted. */
int mk_destroy(mk_handle* h);

const char* mk_status_string(int status);

/* Mid-states of the last step, copied (async on `stream`, device-to-device or
 * device-to-host per `dst`) into dst[bytes]:
 *   MK_STATE_HIDDEN      float[2*n_layers+1][batch][hidden]: index 0 is the
 *                        embedding, 2l+1 the residual after layer l's
 *                        attention block, 2l+2 after its MLP block
 *   MK_STATE_ROUTER      float[n_layers][batch][n_experts] router logits (MoE)
 *   MK_STATE_SELECTION   int32[n_layers][batch][top_k] chosen experts (MoE)
 *   MK_STATE_SEL_WEIGHT  float[n_layers][batch][top_k] their weights (MoE)
 *   MK_STATE_EXPERT_COUNT int32[n_layers] distinct experts used (MoE)
 *   MK_STATE_TRACE       uint64[n_instr][8] per-instruction %globaltimer stamps
 *                        (ns) of the last step, in mk_plan_copy order: consumer
 *                        start, dependency satisfied, compute done, producer's
 *                        first copy issued, prologue done, first stage landed,
 *                        last stage consumed, producer's last copy issued.
 *                        Only for handles created with the environment variable
 *                        MK_TRACE=1 (0 bytes otherwise).
 *   MK_STATE_COUNTERS    uint32[mk_plan_n_counters] the dependency counters
 *                        after the last step: each has counted epoch x its
 *                        target (mk_plan_counter_targets), epoch being the steps run
 *                        since the handle was made or a failing step's status
 *                        was read (that read clears them) */
enum {
  MK_STATE_HIDDEN = 0,
  MK_STATE_ROUTER = 1,
  MK_STATE_SELECTION = 2,
  MK_STATE_SEL_WEIGHT = 3,
  MK_STATE_EXPERT_COUNT = 4,
  MK_STATE_TRACE = 5,
  MK_STATE_COUNTERS = 6
};
int mk_read_state(mk_handle* h, int which, void* dst, size_t bytes, void* stream);

/* Bytes of the mid-state `which` (0 if the model has none). */
size_t mk_state_bytes(const mk_handle* h, int which);

/*
 * mk_decode_step_noalloc: one decode step that allocates no device memory.
 * (No counterpart in the paper: an addition for callers that cannot call
 * cudaMalloc where they decode, e.g. a plugin inside another engine that owns
 * every device byte, or a real-time path that must not enter the allocator.)
 *
 * Same model, weights, cache and per-step arguments as mk_create followed by
 * mk_decode_step, and the same kernel, but every byte of library state lives
 * in one static device array of 8 MiB that each GPU loading the library holds
 * until the process exits.  A model whose state (instruction lists, counters,
 * activations, RoPE table) needs more returns MK_ERR_UNSUPPORTED.
 *   - The first call on a device resolves the array's address there
 *     (cudaGetSymbolAddress with that device current).
 *   - Each call clears the counters and status words it uses, uploads the
 *     instruction lists from temporary host memory, launches on `stream` and
 *     then synchronises `stream` so that it can return the device-side status
 *     (MK_OK, MK_ERR_RANGE, MK_ERR_DEVICE_TIMEOUT).
 *   - All calls share the array, which keeps the last call's contents: calls
 *     that overlap on the GPU (other streams, other host threads) race.
 */
int mk_decode_step_noalloc(const mk_model_desc* desc, const mk_weights* weights, const mk_kv* kv,
                           const int32_t* tokens, const int32_t* positions, const int32_t* seq_lens, void* stream,
                           float* out_logits);

/* ---- host-only lowering (no GPU needed) ---------------------------------- */

/* One instruction of a per-SM list (8 x int32); see mk_plan_* below. */
typedef struct mk_instr {
  int32_t op_layer;   /* op | layer << 8 */
  int32_t wait_idx;   /* counter waited on, -1 none */
  int32_t wait_count; /* producers per step the wait needs */
  int32_t sig_idx;    /* counter bumped on completion, -1 none */
  int32_t a, b, c, d; /* op arguments */
} mk_instr;

typedef struct mk_plan mk_plan;

/* Lower `desc` for `n_sm` SMs on the host (no CUDA call).  Same validation
 * and the same lists that mk_create builds for a device with n_sm SMs. */
int mk_plan_create(const mk_model_desc* desc, int n_sm, mk_plan** out);
int mk_plan_n_sm(const mk_plan* p);
int mk_plan_n_counters(const mk_plan* p);
/* offsets: int32[n_sm+1] (SM s owns instructions [offsets[s], offsets[s+1])). */
int mk_plan_n_instrs(const mk_plan* p);
int mk_plan_copy(const mk_plan* p, mk_instr* instrs, int32_t* offsets);
/* Per-step producers of each counter: int32[n_counters]. */
int mk_plan_counter_targets(const mk_plan* p, int32_t* targets);
/* Attention schedule: `chunk` = positions per unit (one ring stage of K and
 * one of V), `n_chunks` = slots (one per SM per layer; also the most pieces a
 * (sequence, KV head, head group) row is cut into). */
int mk_plan_attn_chunk(const mk_plan* p, int32_t* chunk, int32_t* n_chunks);
/* The attention pieces the kernel derives for one step from `seq_lens`
 * (host int32[batch]): every row (sequence b, KV head, head group) covers
 * positions 0..seq_lens[b] in units of `chunk` positions, and the units of
 * all rows, in row order, are dealt to the slots as equal contiguous runs.
 * Writes up to max_pieces records of 7 int32 (slot, b, row, first unit,
 * end unit, index of the piece within its row, pieces of the row) to `out`
 * and the total count to *n_out; MK_ERR_INVALID_ARG when it exceeds
 * max_pieces, MK_ERR_RANGE for a length outside [0, max_ctx). */
int mk_plan_attn_pieces(const mk_plan* p, const int32_t* seq_lens, int32_t* out, int32_t max_pieces,
                        int32_t* n_out);
int mk_plan_destroy(mk_plan* p);

#ifdef __cplusplus
}
#endif
#endif
