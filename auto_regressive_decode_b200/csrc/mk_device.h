// Kernel parameters shared by the C ABI (host) and the persistent kernel.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mk_internal.h"

namespace mk {

struct LayerPtrs {
  const uint16_t *attn_norm, *wq, *wk, *wv, *q_norm, *k_norm, *wo, *mlp_norm;
  const uint16_t *w_gate, *w_up, *w_down, *router;
};

struct Params {
  // shape
  int L, H, nq, nkv, hd, I, V, B, T, qk_norm;
  int tc;  // the tensor-core kernel (batch > 1 or MoE)
  float eps;
  int chunk, n_chunks;
  // weights (device)
  const uint16_t* embed;
  const uint16_t* final_norm;
  const uint16_t* lm_head;
  const LayerPtrs* layers;  // [L]
  uint16_t* kc;             // [L][B][nkv][T][hd], or paged: [L][n_pages][nkv][page][hd]
  uint16_t* vc;
  const int32_t* bt;        // paged cache: block table [B][bt_stride], else nullptr
  int page, n_pages, bt_stride;
  const float2* rope;       // [T][hd/2] (cos, sin)
  // batch > 1: TMA tensor maps (CUtensorMap, 128 bytes each) of every weight
  // matrix: [layer][wq wk wv wo w_gate w_up w_down], then the LM head, the K
  // cache and the V cache
  const uint8_t* tmaps;
  // batch-1 kernel: 2-D TMA maps of every weight matrix, kB1BoxHeights per
  // matrix (boxes of kB1Chunk columns x 64, 32, 16, 8, 4, 2, 1 rows): [layer][wq wk wv
  // wo w_gate w_up w_down], then the LM head
  const uint8_t* tmaps_b1;
  // library scratch (device)
  float* xres;              // [2L+1][B][H]
  float* qkv;               // [B][nq*hd + 2*nkv*hd]
  float* attn;              // [B][nq*hd]
  float* act;               // [B][I]
  // tensor-core kernel: the inputs of o_proj and down, bf16 (the mma operand type)
  uint16_t* attn_bf;        // [B][nq*hd]
  uint16_t* act_bf;         // [B][I]
  float* part_o;            // [B][nq][n_chunks][hd]
  float* part_ml;           // [B][nq][n_chunks][2]
  // MoE: E experts, top-k, expert SwiGLU width Ie; router logits and routing
  // of every layer of the step (kept for mk_read_state)
  int E, topk, Ie;
  float* moe_router;        // [L][B][E]
  int32_t* moe_sel;         // [L][B][topk] picked experts, best first
  float* moe_selw;          // [L][B][topk] their weights
  int32_t* moe_count;       // [L] distinct picked experts
  uint16_t* moe_act;        // [slots][B][Ie] SwiGLU outputs of the picked experts times the
                            // sequence's routing weight (0 if it did not pick the slot), bf16
  uint32_t* counters;       // [n_counters]
  uint32_t* tickets;        // [L][B][nkv]
  const mk_instr* instrs;
  const int32_t* offsets;   // [n_sm + 1]
  int* status;              // [0] code, [1] detail, [2] block
  // per step
  const int32_t* tokens;
  const int32_t* positions;
  const int32_t* seq_lens;
  float* logits;            // [B][V]
  unsigned long long* argmax;  // greedy decoding: [B] packed (logit, token) maxima, or nullptr
  uint32_t epoch;
  uint64_t timeout_ns;
  uint64_t* trace;          // [n_instr][kTraceStamps] timestamps, or nullptr
};

// Encode the 3-D tensor maps of the batch > 1 kernel (one per weight matrix,
// then the K and V caches) into host memory `out` (kTmapsPerLayer * L + 3
// maps of 128 bytes).  Returns cudaErrorInvalidValue when the driver rejects a
// map (alignment, sizes).
cudaError_t encode_tmaps(const mk_model_desc& d, const mk_weights& w, const mk_kv& kv, uint8_t* out);

// Maps of the batch-1 kernel's row-stationary tiles (kB1MapsPerLayer * L + 2
// maps of 128 bytes) into host memory `out`.
cudaError_t encode_tmaps_b1(const mk_model_desc& d, const mk_weights& w, uint8_t* out);
inline size_t n_tmaps_b1(const mk_model_desc& d) { return (size_t)kB1MapsPerLayer * d.n_layers + kB1BoxHeights; }

// Dynamic shared memory of one CTA.
size_t kernel_smem_bytes(bool batched);
cudaError_t kernel_prepare();  // set both kernels' shared-memory limits
cudaError_t kernel_occupancy(int* blocks_per_sm, bool batched);
cudaError_t launch_step(const Params& p, int n_blocks, cudaStream_t stream);

}  // namespace mk
