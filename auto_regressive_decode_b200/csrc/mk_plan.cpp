// Host scheduler: lowers one decode step of a model into per-SM instruction
// lists with producer/consumer dependency counters.
//
// ForgeMegakernel (arXiv 2609.12379, abstract) names the two structural
// properties followed here: "a fine-grained instruction stream for each SM"
// and "dependency counters replacing the global synchronization".  The
// lowering below is this library's own: every GEMV is cut into one contiguous
// row range per SM (so each SM streams the same number of weight bytes per
// op), attention gets one slot per SM whose share of the step's cached
// positions the kernel computes from the sequence lengths (equal for every
// SM), and every instruction waits on exactly one counter: the one bumped by
// the op it reads.
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "mk_internal.h"

struct mk_plan {
  mk_model_desc d;
  int n_sm;
  int chunk, n_chunks;
  std::vector<std::vector<mk_instr>> lists;
  std::vector<int32_t> targets;
};

namespace mk {

int validate_desc(const mk_model_desc* d) {
  if (!d) return MK_ERR_INVALID_ARG;
  if (d->n_layers <= 0 || d->hidden <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0 ||
      d->vocab <= 0 || d->batch <= 0 || d->max_ctx <= 0 || d->n_layers > (1 << 20))
    return MK_ERR_INVALID_ARG;
  if (!(d->rms_eps >= 0.0f) || !(d->rope_theta > 0.0f)) return MK_ERR_INVALID_ARG;
  if (d->n_experts < 0 || d->ffn_dim < 0) return MK_ERR_INVALID_ARG;
  if (d->n_q_heads % d->n_kv_heads) return MK_ERR_UNSUPPORTED;
  const int g = d->n_q_heads / d->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return MK_ERR_UNSUPPORTED;
  if (d->head_dim != 64 && d->head_dim != 128) return MK_ERR_UNSUPPORTED;
  if (d->batch > kMaxBatch) return MK_ERR_UNSUPPORTED;
  const int qd = d->n_q_heads * d->head_dim;
  if (d->n_experts) {
    // MoE runs on the tensor-core kernel at any batch size
    if (d->top_k <= 0 || d->top_k > d->n_experts || d->expert_ffn_dim <= 0) return MK_ERR_INVALID_ARG;
    if (d->n_experts > kMaxExperts || d->top_k > kMaxTopK || d->batch * d->top_k > kMaxSel) return MK_ERR_UNSUPPORTED;
    const int ks[3] = {d->hidden, qd, d->expert_ffn_dim};
    for (int K : ks)
      if (K % 64) return MK_ERR_UNSUPPORTED;
  } else if (d->ffn_dim <= 0) {
    return MK_ERR_INVALID_ARG;
  }
  // GEMV widths: rows of whole 16-byte vectors (the TMA maps' row pitch)
  const int ks[3] = {d->hidden, qd, d->n_experts ? d->expert_ffn_dim : d->ffn_dim};
  for (int K : ks)
    if (K % 8) return MK_ERR_UNSUPPORTED;
  if ((int64_t)d->max_ctx * d->head_dim > (1ll << 31)) return MK_ERR_UNSUPPORTED;
  if (d->batch > 1 && !d->n_experts) {
    // tensor-core GEMVs: the weight tensor maps view K as blocks of 64 columns
    const int kb[3] = {d->hidden, qd, d->ffn_dim};
    for (int K : kb)
      if (K % 64) return MK_ERR_UNSUPPORTED;
  }
  return MK_OK;
}

namespace {

struct Builder {
  mk_plan* p;
  int emit(int sm, int op, int layer, int wait_idx, int wait_count, int sig_idx, int a, int b, int c = 0, int d = 0) {
    mk_instr in;
    in.op_layer = op | (layer << 8);
    in.wait_idx = wait_idx;
    in.wait_count = wait_count;
    in.sig_idx = sig_idx;
    in.a = a;
    in.b = b;
    in.c = c;
    in.d = d;
    p->lists[sm].push_back(in);
    return 1;
  }
  // Rows [0, N) of one op split evenly over the SMs, each SM's share cut
  // into equal instructions of at most max_rows rows.  Only the last
  // instruction of an SM's share signals (its release covers the earlier
  // ones' outputs), so the counter's per-step target is the number of SMs
  // holding rows of the op, which this returns.
  int rows_op(int op, int layer, int N, int wait_idx, int wait_count, int sig_idx) {
    int n_sig = 0;
    const int n_sm = p->n_sm;
    const int max_rows = batched(p->d) ? batched_max_rows(op) : b1_max_rows(op);
    // batch > 1: row ranges start at multiples of kBBoxRows (a TMA box
    // never reaches into another SM's rows); batch 1: any row
    const int unit = batched(p->d) ? kBBoxRows : 1;
    const int64_t NU = (N + unit - 1) / unit;
    for (int s = 0; s < n_sm; ++s) {
      const int64_t u0 = NU * s / n_sm, u1 = NU * (s + 1) / n_sm;
      if (u0 >= u1) continue;
      const int64_t units = u1 - u0, cap = std::max(1, max_rows / unit);
      const int64_t n_i = (units + cap - 1) / cap;
      for (int64_t i = 0; i < n_i; ++i) {
        const int r0 = (int)std::min<int64_t>(N, (u0 + units * i / n_i) * unit);
        const int r1 = (int)std::min<int64_t>(N, (u0 + units * (i + 1) / n_i) * unit);
        emit(s, op, layer, wait_idx, wait_count, i + 1 == n_i ? sig_idx : -1, r0, r1);
      }
      ++n_sig;
    }
    return n_sig;
  }
};

// Positions per attention unit: one ring stage of K (and one of V).
// MK_ATTN_UNIT (1 .. that) sets a smaller unit, for tests of ragged pieces.
int attn_unit(const mk_model_desc* d) {
  const int P = attn_stage_positions(d->head_dim);
  const char* env = getenv("MK_ATTN_UNIT");
  if (env && atoi(env) > 0) return std::min(atoi(env), P);
  return P;
}

}  // namespace

int build_plan(const mk_model_desc* d, int n_sm, mk_plan* p) {
  p->d = *d;
  p->n_sm = n_sm;
  p->lists.assign(n_sm, {});
  const int L = d->n_layers, H = d->hidden, hd = d->head_dim;
  const int qd = d->n_q_heads * hd, kvd = d->n_kv_heads * hd;
  p->targets.assign(n_counters(L), 0);
  // attention: one slot per SM per layer; a row's pieces are at most n_sm
  p->chunk = attn_unit(d);
  p->n_chunks = n_sm;
  // the merging CTA stages (m, l) of every (query head of the group, piece) in
  // its kRedFloats-float reduction buffer
  if (2 * attn_heads_per_instr(d->n_q_heads / d->n_kv_heads) * p->n_chunks > kRedFloats) return MK_ERR_UNSUPPORTED;
  Builder b{p};

  // x0 = embedding rows, hidden dimension split over the SMs
  int n_embed = 0;
  const int c_embed = counter_embed(L);
  for (int s = 0; s < n_sm; ++s) {
    int r0 = (int)((int64_t)H * s / n_sm), r1 = (int)((int64_t)H * (s + 1) / n_sm);
    if (r0 < r1) n_embed += b.emit(s, OP_EMBED, 0, -1, 0, c_embed, r0, r1);
  }
  p->targets[c_embed] = n_embed;

  int prev_idx = c_embed, prev_count = n_embed;
  for (int l = 0; l < L; ++l) {
    const int cq = counter_index(l, C_QKV), ca = counter_index(l, C_ATTN), co = counter_index(l, C_OPROJ);
    const int cg = counter_index(l, C_GATEUP), cd = counter_index(l, C_DOWN);
    // rows of wq | wk | wv concatenated; an instruction may span matrices
    int n_qkv = b.rows_op(OP_QKV, l, qd + 2 * kvd, prev_idx, prev_count, cq);
    p->targets[cq] = n_qkv;
    // attention: slot j = SM j; the kernel deals the step's units to the slots
    const int group = d->n_q_heads / d->n_kv_heads, nhg = group / attn_heads_per_instr(group);
    for (int s = 0; s < n_sm; ++s) b.emit(s, OP_ATTN, l, cq, n_qkv, ca, s, n_sm, 0, 0);
    p->targets[ca] = d->batch * d->n_kv_heads * nhg;  // one bump per merged (sequence, KV head, head group)
    int n_o = b.rows_op(OP_OPROJ, l, H, ca, p->targets[ca], co);
    p->targets[co] = n_o;
    if (d->n_experts) {
      // router rows; one expert gate/up slot per SM; down by output rows
      const int cr = counter_index(l, C_ROUTER), ceg = counter_index(l, C_EXP_GATEUP);
      const int ced = counter_index(l, C_EXP_DOWN);
      int n_r = b.rows_op(OP_ROUTER, l, d->n_experts, co, n_o, cr);
      p->targets[cr] = n_r;
      for (int s = 0; s < n_sm; ++s) b.emit(s, OP_EXP_GATEUP, l, cr, n_r, ceg, s, n_sm, 0, 0);
      p->targets[ceg] = n_sm;
      int n_ed = b.rows_op(OP_EXP_DOWN, l, H, ceg, n_sm, ced);
      p->targets[ced] = n_ed;
      prev_idx = ced;
      prev_count = n_ed;
      continue;
    }
    int n_gu = b.rows_op(OP_GATEUP, l, d->ffn_dim, co, n_o, cg);
    p->targets[cg] = n_gu;
    int n_dn = b.rows_op(OP_DOWN, l, H, cg, n_gu, cd);
    p->targets[cd] = n_dn;
    prev_idx = cd;
    prev_count = n_dn;
  }
  const int c_lm = counter_lmhead(L);
  p->targets[c_lm] = b.rows_op(OP_LMHEAD, L, d->vocab, prev_idx, prev_count, c_lm);
  // Host-made fault for tests of the failure path (never set in normal use):
  // MK_FAULT_INJECT=wait makes SM 0's first instruction wait on a counter no
  // instruction ever raises far enough, so every bounded wait must run out.
  const char* fault = getenv("MK_FAULT_INJECT");
  if (fault && strcmp(fault, "wait") == 0 && !p->lists[0].empty()) {
    p->lists[0][0].wait_idx = c_lm;
    p->lists[0][0].wait_count = p->targets[c_lm] + 1;
  }
  return MK_OK;
}

}  // namespace mk

// ---- C ABI: host-only lowering ---------------------------------------------------

extern "C" int mk_plan_create(const mk_model_desc* desc, int n_sm, mk_plan** out) {
  if (!out || n_sm <= 0) return MK_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = mk::validate_desc(desc);
  if (rc) return rc;
  mk_plan* p = new (std::nothrow) mk_plan();
  if (!p) return MK_ERR_INVALID_ARG;
  rc = mk::build_plan(desc, n_sm, p);
  if (rc) {
    delete p;
    return rc;
  }
  *out = p;
  return MK_OK;
}

extern "C" int mk_plan_n_sm(const mk_plan* p) { return p ? p->n_sm : MK_ERR_INVALID_ARG; }

extern "C" int mk_plan_n_counters(const mk_plan* p) { return p ? (int)p->targets.size() : MK_ERR_INVALID_ARG; }

extern "C" int mk_plan_n_instrs(const mk_plan* p) {
  if (!p) return MK_ERR_INVALID_ARG;
  size_t n = 0;
  for (auto& l : p->lists) n += l.size();
  return (int)n;
}

extern "C" int mk_plan_copy(const mk_plan* p, mk_instr* instrs, int32_t* offsets) {
  if (!p || !instrs || !offsets) return MK_ERR_INVALID_ARG;
  int32_t o = 0;
  for (int s = 0; s < p->n_sm; ++s) {
    offsets[s] = o;
    memcpy(instrs + o, p->lists[s].data(), p->lists[s].size() * sizeof(mk_instr));
    o += (int32_t)p->lists[s].size();
  }
  offsets[p->n_sm] = o;
  return MK_OK;
}

extern "C" int mk_plan_counter_targets(const mk_plan* p, int32_t* targets) {
  if (!p || !targets) return MK_ERR_INVALID_ARG;
  memcpy(targets, p->targets.data(), p->targets.size() * sizeof(int32_t));
  return MK_OK;
}

extern "C" int mk_plan_attn_chunk(const mk_plan* p, int32_t* chunk, int32_t* n_chunks) {
  if (!p || !chunk || !n_chunks) return MK_ERR_INVALID_ARG;
  *chunk = p->chunk;
  *n_chunks = p->n_chunks;
  return MK_OK;
}

extern "C" int mk_plan_attn_pieces(const mk_plan* p, const int32_t* seq_lens, int32_t* out, int32_t max_pieces,
                                   int32_t* n_out) {
  if (!p || !seq_lens || !n_out || max_pieces < 0 || (max_pieces > 0 && !out)) return MK_ERR_INVALID_ARG;
  for (int b = 0; b < p->d.batch; ++b)
    if (seq_lens[b] < 0 || seq_lens[b] >= p->d.max_ctx) return MK_ERR_RANGE;
  const int group = p->d.n_q_heads / p->d.n_kv_heads;
  mk::AttnSched sc;
  mk::attn_sched_init(sc, seq_lens, p->d.batch, p->d.n_kv_heads * (group / mk::attn_heads_per_instr(group)), p->chunk,
                  p->n_chunks);
  int n = 0;
  for (int j = 0; j < sc.n_slots; ++j) {
    for (int64_t g = mk::attn_slot_begin(sc, j), g1 = mk::attn_slot_begin(sc, j + 1); g < g1;) {
      const mk::AttnPiece pc = mk::attn_piece_at(sc, g, j);
      if (n < max_pieces) {
        int32_t* o = out + (size_t)n * 7;
        o[0] = j;
        o[1] = pc.b;
        o[2] = pc.row;
        o[3] = pc.ua;
        o[4] = pc.ub;
        o[5] = pc.slot_in_row;
        o[6] = pc.n_pieces;
      }
      ++n;
      g += pc.ub - pc.ua;
    }
  }
  *n_out = n;
  return n <= max_pieces ? MK_OK : MK_ERR_INVALID_ARG;
}

extern "C" int mk_plan_destroy(mk_plan* p) {
  delete p;
  return MK_OK;
}
