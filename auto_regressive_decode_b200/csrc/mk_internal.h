// Internal definitions shared by the host scheduler (mk_plan.cpp), the C ABI
// (mk_api.cu) and the persistent kernel (mk_kernel.cu).
#pragma once

#include <stdint.h>

#include "../../include/mk.h"

#if defined(__CUDACC__)
#define MK_HD __host__ __device__ __forceinline__
#else
#define MK_HD inline
#endif

namespace mk {

// ---- instruction ops (low 8 bits of mk_instr::op_layer) --------------------
enum Op : int32_t {
  OP_NOP = 0,
  OP_EMBED = 1,    // a,b: hidden slice [a,b) of x0 = embed[token]
  OP_QKV = 2,      // a,b: rows of wq|wk|wv concatenated; RMSNorm(x_{2l}) prologue
  OP_ATTN = 3,     // a: sequence, b: kv head, c: chunk, d: head group; last chunk of (a,b,d) merges
  OP_OPROJ = 4,    // a,b: rows of wo; x_{2l+1} = x_{2l} + wo . attn
  OP_GATEUP = 5,   // a,b: rows of w_gate/w_up; act = silu(g) * u; RMSNorm(x_{2l+1}) prologue
  OP_DOWN = 6,     // a,b: rows of w_down; x_{2l+2} = x_{2l+1} + w_down . act
  OP_LMHEAD = 7,   // a,b: vocabulary rows; RMSNorm(x_{2L}) prologue
  OP_ROUTER = 8,   // a: sequence; router logits, top-k, expert list (MoE)
  OP_EXP_GATEUP = 9,  // a,b: rows of every used expert's gate/up (MoE)
  OP_EXP_DOWN = 10,   // a,b: rows of every used expert's down + weighted combine (MoE)
};

MK_HD int op_of(int32_t op_layer) { return op_layer & 0xFF; }
MK_HD int layer_of(int32_t op_layer) { return op_layer >> 8; }

// ---- pipeline geometry -----------------------------------------------------
constexpr int kConsumerWarps = 8;                      // compute warps
constexpr int kConsumerThreads = kConsumerWarps * 32;  // 256
constexpr int kThreads = kConsumerThreads + 32;        // + one producer warp
constexpr int kStageBytes = 32 * 1024;                 // one ring slot
constexpr int kStages = 6;                             // ring depth (192 KB), batch-1 kernel
constexpr int kStagesBatched = 5;                      // ring depth of the tensor-core kernel
// tensor-core kernel: bf16 inputs of o_proj / down / expert down staged in
// shared memory, kXsSlots chunks of [kMaxBatch][kBChunk] at a padded pitch
constexpr int kXsPitchBytes = 1024 * 2 + 16;
constexpr int kXsSlots = 3;
constexpr int kRedFloats = 4096;                       // cross-warp reduction buffer
constexpr int kMaxBatch = 8;
constexpr int kMaxGroup = 8;                           // query heads per KV head
constexpr int kMaxHeadDim = 128;
constexpr int kTraceStamps = 8;                        // per-instruction trace words

// ---- dependency counters -----------------------------------------------------
// Each counter is bumped once per producing instruction per step; a waiter
// needs epoch * producers.  Per layer: QKV, ATTN (one per merged (seq, kv head)),
// OPROJ, GATEUP / ROUTER, DOWN / EXP_GATEUP, EXP_DOWN.
enum CounterSlot : int32_t {
  C_QKV = 0,
  C_ATTN = 1,
  C_OPROJ = 2,
  C_GATEUP = 3,
  C_DOWN = 4,
  C_ROUTER = 5,
  C_EXP_GATEUP = 6,
  C_EXP_DOWN = 7,
  C_PER_LAYER = 8
};
inline int counter_index(int layer, int slot) { return layer * C_PER_LAYER + slot; }
// global counters after the per-layer block
inline int counter_embed(int n_layers) { return n_layers * C_PER_LAYER; }
inline int counter_lmhead(int n_layers) { return n_layers * C_PER_LAYER + 1; }
inline int n_counters(int n_layers) { return n_layers * C_PER_LAYER + 2; }

// ---- batch-1 GEMV tiling (host and device agree on it) -----------------------
// Row-stationary tiles: an instruction owns `lines` weight rows (rows x matrices;
// gate/up pairs count twice) and streams K in chunks of kB1Chunk columns.  A
// stage holds every line of the instruction for `nc` consecutive chunks, each
// line a 512-byte row of shared memory, moved by 2-D TMA boxes of 64 down to 1
// rows (no swizzle; few, tall boxes: each box costs the copy engine a fixed
// time).  Consumer warps keep the partial dot products of their lines in
// registers across all chunks: one warp reduction per instruction, none per stage.
constexpr int kB1Chunk = 256;          // columns per chunk (the TMA box width)
constexpr int kB1LineBytes = kB1Chunk * 2;
constexpr int kB1MaxLines = 64;        // lines per instruction (64 x 512 B = one stage)
constexpr int kB1TallestBox = 64;      // box maps of 64, 32, 16, 8, 4, 2 and 1 rows per matrix
constexpr int kB1BoxHeights = 7;
constexpr int kB1MapsPerLayer = 7 * kB1BoxHeights;  // wq wk wv wo w_gate w_up w_down
// The input vector of a batch-1 GEMV sits in shared memory (fp32, the norm's
// gain applied) in pieces of at most kB1XPieceFloats columns, loaded once per
// piece with one round trip to L2: the same op's next instruction on the SM
// reuses it, and a K longer than a piece reloads mid-instruction.
constexpr int kB1XPieceFloats = 6144;
// rows (gate/up: neurons) per instruction; a gate/up instruction of more than
// kB1MaxLines / 2 neurons streams its gate rows and its up rows as two groups
MK_HD int b1_max_rows(int op) { return kB1MaxLines; }
// chunks per stage: as many as fill a stage with the instruction's lines
MK_HD int b1_chunks_per_stage(int lines) { return lines > 32 ? 1 : (lines > 16 ? 2 : 4); }
// chunks per input piece: whole stages
MK_HD int b1_piece_chunks(int ncs) { return kB1XPieceFloats / kB1Chunk / ncs * ncs; }
static_assert(kB1MaxLines * kB1LineBytes == kStageBytes, "a stage of 64 lines fills a ring slot");

// ---- batch > 1 GEMV (tensor cores) -------------------------------------------------
// A stage is one tile of 16 A-operand rows (16 weight rows, or 8 gate rows over
// the same 8 up rows) for one chunk of kBChunk input columns, moved as two TMA
// boxes of kBBoxRows rows each.  A weight matrix [N][K] is viewed by its tensor
// map as a 3-D tensor (64 columns, N rows, K/64 column blocks), so that a box
// lands as [column block][row][64] with 128-byte rows swizzled (16-byte chunk
// c of line L stored at chunk c ^ (L & 7)): the eight row reads of an ldmatrix
// phase hit distinct bank groups.  An instruction streams chunk by chunk, and
// tile by tile within a chunk; row ranges are cut at multiples of kBBoxRows.
constexpr int kBChunk = 1024;                        // input columns per stage
constexpr int kBBoxRows = 8;                         // weight rows per TMA box
constexpr int kBBoxBytes = kBBoxRows * kBChunk * 2;  // 16 KB
constexpr int kBatchedMaxRows = 128;                 // rows per instruction: 8 tiles of 16
constexpr int kBatchedMaxRowsGated = 96;             // gate/up: 12 tiles of 8 neurons
constexpr int kBatchedMaxRowsLongK = 64;             // o_proj, down, expert down: 4 tiles of 16
MK_HD int batched_max_rows(int op) {
  return op == OP_GATEUP ? kBatchedMaxRowsGated
                         : (op == OP_OPROJ || op == OP_DOWN || op == OP_EXP_DOWN ? kBatchedMaxRowsLongK : kBatchedMaxRows);
}
constexpr int kTmapsPerLayer = 8;  // wq wk wv wo w_gate w_up w_down router (then LM head, K cache, V cache)
MK_HD int btile_rows(bool gated) { return gated ? 8 : 16; }
// The tensor-core kernel runs every batch > 1 model and every MoE model.
MK_HD bool batched(const mk_model_desc& d) { return d.batch > 1 || d.n_experts > 0; }

// ---- mixture of experts ------------------------------------------------------------
// Router GEMV over the experts, top-k per sequence, then the distinct picked
// experts ("slots", ascending expert index).  Gate/up work is (slot, 8-neuron
// tile) units dealt evenly to one instruction per SM; down is split by output
// rows and runs over all slots, the routing weights folded into its inputs.
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
constexpr int kMaxSel = 64;  // distinct experts of one step: at most batch * top_k
MK_HD int moe_slots(int n_experts, int batch, int top_k) {
  return n_experts < batch * top_k ? n_experts : batch * top_k;
}

// Even deal of U units to n slots (n cut to U when U < n, so that every slot
// in use holds a unit): the first unit of slot j.
MK_HD int64_t even_begin(int64_t U, int n, int j) {
  const int m = U < n ? (int)U : n;
  return j >= m ? U : U * j / m;
}

// ---- attention split -------------------------------------------------------------
// Query heads one attention instruction handles: a KV head with more query
// heads than this is split into head groups, each a separate instruction
// over the same cache chunk (keeps the per-thread accumulators in registers).
MK_HD int attn_heads_per_instr(int group) { return group > 4 ? 4 : group; }

// The merging piece of an attention row loads the partial outputs of its
// first kMergeAhead pieces together with their (m, l) pairs.
constexpr int kMergeAhead = 24;

// Positions of K (or V) that fit one ring slot.
MK_HD int attn_stage_positions(int head_dim) { return kStageBytes / (head_dim * 2); }

// ---- attention schedule (computed on the device from each step's seq_lens) --------
// A row is (sequence b, KV head, head group); its work is the positions
// 0..S_b (S_b cached ones and the new token) in units of `unit` positions,
// u_b = S_b / unit + 1 units.  Rows are ordered (b, KV head, head group) and
// the U units of all rows are dealt to n = min(n_slots, U) slots as contiguous
// runs [U j / n, U (j + 1) / n): every slot streams the same number of units
// (to within one), whatever the lengths.  A slot's run is cut into pieces at row
// boundaries; each piece writes a partial (o, m, l) and the last piece of a
// row to finish merges the row's pieces in slot order.
struct AttnSched {
  int unit, n_slots, rows_per_seq, B;
  int64_t U;
  int u[kMaxBatch];          // units per row of sequence b
  int64_t base[kMaxBatch + 1];  // first global unit of sequence b
};

struct AttnPiece {
  int b, row;          // sequence, row within the sequence (KV head * head groups + head group)
  int ua, ub;          // units [ua, ub) of the row
  int slot_in_row;     // index of this piece among the row's pieces
  int n_pieces;        // pieces of the row
};

MK_HD void attn_sched_init(AttnSched& s, const int32_t* seq_lens, int B, int rows_per_seq, int unit, int n_slots) {
  s.unit = unit;
  s.n_slots = n_slots;
  s.rows_per_seq = rows_per_seq;
  s.B = B;
  s.base[0] = 0;
  for (int b = 0; b < kMaxBatch; ++b) {
    s.u[b] = b < B ? seq_lens[b] / unit + 1 : 0;
    s.base[b + 1] = s.base[b] + (int64_t)rows_per_seq * s.u[b];
  }
  s.U = s.base[B];
  // fewer units than slots: one unit each for the first U slots, none after,
  // so that every slot in use holds at least one unit
  if (s.U < s.n_slots) s.n_slots = (int)s.U;
}

// First global unit of slot j (U for j >= the slots in use).
MK_HD int64_t attn_slot_begin(const AttnSched& s, int j) { return j >= s.n_slots ? s.U : s.U * j / s.n_slots; }

// The slot holding global unit g (0 <= g < U).
MK_HD int attn_slot_of(const AttnSched& s, int64_t g) { return (int)(((g + 1) * s.n_slots - 1) / s.U); }

// The piece of slot j that starts at global unit g (g < end of slot j).
MK_HD AttnPiece attn_piece_at(const AttnSched& s, int64_t g, int j) {
  AttnPiece pc;
  int b = 0;
  while (b + 1 < s.B && s.base[b + 1] <= g) ++b;
  const int64_t off = g - s.base[b];
  pc.b = b;
  pc.row = (int)(off / s.u[b]);
  pc.ua = (int)(off % s.u[b]);
  const int64_t left = attn_slot_begin(s, j + 1) - g;
  pc.ub = (int)((int64_t)(s.u[b] - pc.ua) < left ? s.u[b] : pc.ua + left);
  const int64_t first = s.base[b] + (int64_t)pc.row * s.u[b];
  const int s0 = attn_slot_of(s, first);
  pc.slot_in_row = j - s0;
  pc.n_pieces = attn_slot_of(s, first + s.u[b] - 1) - s0 + 1;
  return pc;
}

}  // namespace mk
