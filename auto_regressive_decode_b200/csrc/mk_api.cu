// C ABI of the decode megakernel (declared in include/mk.h).
//
// mk_create validates the model, lowers it (mk_plan.cpp), and allocates one
// device region holding everything the library owns.  mk_decode_step is a
// single cooperative launch with no host synchronisation.  Errors found on the
// device are recorded in a status word that mk_get_status reads and clears.
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>
#include <vector>

#include "mk_device.h"
#include "mk_internal.h"

namespace mk {
int validate_desc(const mk_model_desc* d);
int build_plan(const mk_model_desc* d, int n_sm, mk_plan* p);
}  // namespace mk

struct mk_plan;  // defined in mk_plan.cpp
extern "C" int mk_plan_create(const mk_model_desc*, int, mk_plan**);
extern "C" int mk_plan_n_instrs(const mk_plan*);
extern "C" int mk_plan_copy(const mk_plan*, mk_instr*, int32_t*);
extern "C" int mk_plan_n_counters(const mk_plan*);
extern "C" int mk_plan_attn_chunk(const mk_plan*, int32_t*, int32_t*);
extern "C" int mk_plan_destroy(mk_plan*);

struct mk_handle {
  mk_model_desc d;
  mk::Params p;
  int n_sm;
  int device;
  int n_counters;
  size_t n_tickets;
  void* region;
  size_t region_bytes;
  size_t n_instr;
  uint32_t epoch;
  // greedy decoding loop: the steps' tokens and lengths, per-sequence arg-max, logits
  int32_t* loop_tok;
  int32_t* loop_len;
  unsigned long long* amax;
  float* loop_logits;
};

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  }
};

}  // namespace

extern "C" const char* mk_status_string(int s) {
  switch (s) {
    case MK_OK: return "ok";
    case MK_ERR_INVALID_ARG: return "invalid argument";
    case MK_ERR_UNSUPPORTED: return "unsupported shape, alignment or device";
    case MK_ERR_CUDA: return "CUDA runtime error";
    case MK_ERR_DEVICE_TIMEOUT: return "in-kernel wait timed out";
    case MK_ERR_RANGE: return "token, position or sequence length out of range";
    default: return "unknown status";
  }
}

extern "C" int mk_create(const mk_model_desc* desc, const mk_weights* w, const mk_kv* kv, mk_handle** out) {
  if (!out) return MK_ERR_INVALID_ARG;
  *out = nullptr;
  if (!desc || !w || !kv || !w->layers) return MK_ERR_INVALID_ARG;
  int rc = mk::validate_desc(desc);
  if (rc) return rc;
  const mk_model_desc& d = *desc;
  // pointers: present and 16-byte aligned
  if (!aligned16(w->embed) || !aligned16(w->final_norm) || !aligned16(kv->k) || !aligned16(kv->v))
    return w->embed && w->final_norm && kv->k && kv->v ? MK_ERR_UNSUPPORTED : MK_ERR_INVALID_ARG;
  if (kv->block_table) {  // paged cache: pages hold whole attention stages
    if (kv->page_size <= 0 || kv->n_pages <= 0) return MK_ERR_INVALID_ARG;
    if (kv->page_size % mk::attn_stage_positions(d.head_dim) ||
        (int64_t)d.n_layers * kv->n_pages * d.n_kv_heads * kv->page_size >= (1ll << 31))
      return MK_ERR_UNSUPPORTED;
  }
  if (!d.tied_embeddings && !aligned16(w->lm_head)) return w->lm_head ? MK_ERR_UNSUPPORTED : MK_ERR_INVALID_ARG;
  for (int l = 0; l < d.n_layers; ++l) {
    const mk_layer_weights& lw = w->layers[l];
    const void* need[] = {lw.attn_norm, lw.wq, lw.wk, lw.wv, lw.wo, lw.mlp_norm, lw.w_gate, lw.w_up, lw.w_down};
    for (const void* q : need)
      if (!aligned16(q)) return q ? MK_ERR_UNSUPPORTED : MK_ERR_INVALID_ARG;
    if (d.qk_norm && (!aligned16(lw.q_norm) || !aligned16(lw.k_norm))) return MK_ERR_INVALID_ARG;
    if (d.n_experts && !aligned16(lw.router)) return lw.router ? MK_ERR_UNSUPPORTED : MK_ERR_INVALID_ARG;
  }

  int dev = 0, n_sm = 0, coop = 0, smem_optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MK_ERR_CUDA;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MK_ERR_CUDA;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess) return MK_ERR_CUDA;
  if (cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return MK_ERR_CUDA;
  if (!coop || (size_t)smem_optin < mk::kernel_smem_bytes(mk::batched(d))) return MK_ERR_UNSUPPORTED;
  if (mk::kernel_prepare() != cudaSuccess) return MK_ERR_CUDA;
  int per_sm = 0;
  if (mk::kernel_occupancy(&per_sm, mk::batched(d)) != cudaSuccess) return MK_ERR_CUDA;
  if (per_sm < 1) return MK_ERR_UNSUPPORTED;

  mk_plan* plan = nullptr;
  rc = mk_plan_create(desc, n_sm, &plan);
  if (rc) return rc;
  const int n_instr = mk_plan_n_instrs(plan);
  std::vector<mk_instr> instrs(n_instr > 0 ? n_instr : 1);
  std::vector<int32_t> offsets(n_sm + 1);
  mk_plan_copy(plan, instrs.data(), offsets.data());
  const int n_cnt = mk_plan_n_counters(plan);
  int32_t chunk = 0, n_chunks = 0;
  mk_plan_attn_chunk(plan, &chunk, &n_chunks);
  if (kv->block_table && chunk != mk::attn_stage_positions(d.head_dim)) {  // a stage must not straddle pages
    mk_plan_destroy(plan);
    return MK_ERR_UNSUPPORTED;
  }
  mk_plan_destroy(plan);

  mk_handle* h = new (std::nothrow) mk_handle();
  if (!h) return MK_ERR_INVALID_ARG;
  h->d = d;
  h->n_sm = n_sm;
  h->device = dev;
  h->n_counters = n_cnt;
  h->epoch = 0;
  const int L = d.n_layers, B = d.batch, H = d.hidden, hd = d.head_dim, nq = d.n_q_heads, nkv = d.n_kv_heads;
  const size_t qd = (size_t)nq * hd, kvd = (size_t)nkv * hd;
  const int group = nq / nkv;
  h->n_tickets = (size_t)L * B * nkv * (group / mk::attn_heads_per_instr(group));

  Carve cv;
  const size_t o_xres = cv.take(sizeof(float) * (size_t)(2 * L + 1) * B * H);
  const size_t o_qkv = cv.take(sizeof(float) * (size_t)B * (qd + 2 * kvd));
  const size_t o_attn = cv.take(sizeof(float) * (size_t)B * qd);
  const size_t o_act = cv.take(sizeof(float) * (size_t)B * (d.n_experts ? 1 : d.ffn_dim));
  const int E = d.n_experts, K = d.top_k;
  const size_t o_mr = E ? cv.take(sizeof(float) * (size_t)L * B * E) : 0;
  const size_t o_ms = E ? cv.take(sizeof(int32_t) * (size_t)L * B * K) : 0;
  const size_t o_mw = E ? cv.take(sizeof(float) * (size_t)L * B * K) : 0;
  const size_t o_mc = E ? cv.take(sizeof(int32_t) * (size_t)L) : 0;
  const size_t o_ma = E ? cv.take(sizeof(uint16_t) * (size_t)mk::moe_slots(E, B, K) * B * d.expert_ffn_dim) : 0;
  const size_t o_abf = mk::batched(d) ? cv.take(sizeof(uint16_t) * (size_t)B * qd) : 0;
  const size_t o_xbf = mk::batched(d) && !E ? cv.take(sizeof(uint16_t) * (size_t)B * d.ffn_dim) : 0;
  const size_t o_po = cv.take(sizeof(float) * (size_t)B * nq * n_chunks * hd);
  const size_t o_pml = cv.take(sizeof(float) * (size_t)B * nq * n_chunks * 2);
  const size_t o_cnt = cv.take(sizeof(uint32_t) * (size_t)n_cnt);
  const size_t o_tk = cv.take(sizeof(uint32_t) * h->n_tickets);
  const size_t o_st = cv.take(sizeof(int) * 4);
  const size_t o_ins = cv.take(sizeof(mk_instr) * instrs.size());
  const size_t o_off = cv.take(sizeof(int32_t) * offsets.size());
  const size_t o_lay = cv.take(sizeof(mk::LayerPtrs) * (size_t)L);
  const size_t o_rope = cv.take(sizeof(float2) * (size_t)d.max_ctx * (hd / 2));
  const size_t n_tmaps = (size_t)mk::kTmapsPerLayer * L + 3;  // KV caches always; weights on the tensor-core kernel
  const size_t o_tmap = n_tmaps ? cv.take(128 * n_tmaps) : 0;
  const size_t n_tb1 = mk::batched(d) ? 0 : mk::n_tmaps_b1(d);  // the batch-1 kernel's weight maps
  const size_t o_tb1 = n_tb1 ? cv.take(128 * n_tb1) : 0;
  const char* trace_env = getenv("MK_TRACE");
  const bool tracing = trace_env && atoi(trace_env) > 0;
  const size_t o_trace = tracing ? cv.take(sizeof(uint64_t) * mk::kTraceStamps * instrs.size()) : 0;
  const size_t o_ltok = cv.take(sizeof(int32_t) * B), o_llen = cv.take(sizeof(int32_t) * B);
  const size_t o_amax = cv.take(sizeof(unsigned long long) * B);
  const size_t o_llog = cv.take(sizeof(float) * (size_t)B * d.vocab);
  h->n_instr = tracing ? (size_t)n_instr : 0;
  h->region_bytes = cv.off;
  if (cudaMalloc(&h->region, h->region_bytes) != cudaSuccess) {
    delete h;
    return MK_ERR_CUDA;
  }
  uint8_t* base = static_cast<uint8_t*>(h->region);

  std::vector<mk::LayerPtrs> lp(L);
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights& s = w->layers[l];
    mk::LayerPtrs& t = lp[l];
    t.attn_norm = (const uint16_t*)s.attn_norm;
    t.wq = (const uint16_t*)s.wq;
    t.wk = (const uint16_t*)s.wk;
    t.wv = (const uint16_t*)s.wv;
    t.q_norm = (const uint16_t*)s.q_norm;
    t.k_norm = (const uint16_t*)s.k_norm;
    t.wo = (const uint16_t*)s.wo;
    t.mlp_norm = (const uint16_t*)s.mlp_norm;
    t.w_gate = (const uint16_t*)s.w_gate;
    t.w_up = (const uint16_t*)s.w_up;
    t.w_down = (const uint16_t*)s.w_down;
    t.router = (const uint16_t*)s.router;
  }
  // RoPE table: angle pos * theta^(-2i/hd) in double, stored as fp32 (cos, sin)
  std::vector<float2> rope((size_t)d.max_ctx * (hd / 2));
  for (int pos = 0; pos < d.max_ctx; ++pos)
    for (int i = 0; i < hd / 2; ++i) {
      const double ang = (double)pos * pow((double)d.rope_theta, -2.0 * i / hd);
      rope[(size_t)pos * (hd / 2) + i] = make_float2((float)cos(ang), (float)sin(ang));
    }

  std::vector<uint8_t> tmaps(128 * n_tmaps), tb1(128 * n_tb1);
  cudaError_t te = n_tmaps ? mk::encode_tmaps(d, *w, *kv, tmaps.data()) : cudaSuccess;
  if (te == cudaSuccess && n_tb1) te = mk::encode_tmaps_b1(d, *w, tb1.data());
  if (te != cudaSuccess) {
    cudaFree(h->region);
    delete h;
    return te == cudaErrorInvalidValue ? MK_ERR_UNSUPPORTED : MK_ERR_CUDA;
  }
  bool ok = cudaMemset(base, 0, h->region_bytes) == cudaSuccess &&
            (!n_tmaps || cudaMemcpy(base + o_tmap, tmaps.data(), tmaps.size(), cudaMemcpyHostToDevice) == cudaSuccess) &&
            (!n_tb1 || cudaMemcpy(base + o_tb1, tb1.data(), tb1.size(), cudaMemcpyHostToDevice) == cudaSuccess) &&
            cudaMemcpy(base + o_ins, instrs.data(), sizeof(mk_instr) * instrs.size(), cudaMemcpyHostToDevice) ==
                cudaSuccess &&
            cudaMemcpy(base + o_off, offsets.data(), sizeof(int32_t) * offsets.size(), cudaMemcpyHostToDevice) ==
                cudaSuccess &&
            cudaMemcpy(base + o_lay, lp.data(), sizeof(mk::LayerPtrs) * L, cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(base + o_rope, rope.data(), sizeof(float2) * rope.size(), cudaMemcpyHostToDevice) ==
                cudaSuccess;
  if (!ok) {
    cudaFree(h->region);
    delete h;
    return MK_ERR_CUDA;
  }

  mk::Params& p = h->p;
  memset(&p, 0, sizeof(p));
  p.L = L;
  p.H = H;
  p.nq = nq;
  p.nkv = nkv;
  p.hd = hd;
  p.I = d.ffn_dim;
  p.V = d.vocab;
  p.B = B;
  p.tc = mk::batched(d);
  p.T = d.max_ctx;
  p.qk_norm = d.qk_norm;
  p.eps = d.rms_eps;
  p.chunk = chunk;
  p.n_chunks = n_chunks;
  p.embed = (const uint16_t*)w->embed;
  p.final_norm = (const uint16_t*)w->final_norm;
  p.lm_head = (const uint16_t*)(d.tied_embeddings ? w->embed : w->lm_head);
  p.layers = (const mk::LayerPtrs*)(base + o_lay);
  p.kc = (uint16_t*)kv->k;
  p.vc = (uint16_t*)kv->v;
  if (kv->block_table) {
    p.bt = kv->block_table;
    p.page = kv->page_size;
    p.n_pages = kv->n_pages;
    p.bt_stride = (d.max_ctx + kv->page_size - 1) / kv->page_size;
  }
  p.rope = (const float2*)(base + o_rope);
  p.tmaps = n_tmaps ? base + o_tmap : nullptr;
  p.tmaps_b1 = n_tb1 ? base + o_tb1 : nullptr;
  p.xres = (float*)(base + o_xres);
  p.qkv = (float*)(base + o_qkv);
  p.attn = (float*)(base + o_attn);
  p.act = (float*)(base + o_act);
  p.part_o = (float*)(base + o_po);
  p.part_ml = (float*)(base + o_pml);
  if (E) {
    p.E = E;
    p.topk = K;
    p.Ie = d.expert_ffn_dim;
    p.moe_router = (float*)(base + o_mr);
    p.moe_sel = (int32_t*)(base + o_ms);
    p.moe_selw = (float*)(base + o_mw);
    p.moe_count = (int32_t*)(base + o_mc);
    p.moe_act = (uint16_t*)(base + o_ma);
  }
  p.attn_bf = o_abf ? (uint16_t*)(base + o_abf) : nullptr;
  p.act_bf = o_xbf ? (uint16_t*)(base + o_xbf) : nullptr;
  p.counters = (uint32_t*)(base + o_cnt);
  p.tickets = (uint32_t*)(base + o_tk);
  p.status = (int*)(base + o_st);
  p.instrs = (const mk_instr*)(base + o_ins);
  p.offsets = (const int32_t*)(base + o_off);
  p.timeout_ns = d.wait_timeout_ns ? d.wait_timeout_ns : kDefaultTimeoutNs;
  p.trace = tracing ? (uint64_t*)(base + o_trace) : nullptr;
  h->loop_tok = (int32_t*)(base + o_ltok);
  h->loop_len = (int32_t*)(base + o_llen);
  h->amax = (unsigned long long*)(base + o_amax);
  h->loop_logits = (float*)(base + o_llog);
  *out = h;
  return MK_OK;
}

extern "C" int mk_decode_step(mk_handle* h, const int32_t* tokens, const int32_t* positions, const int32_t* seq_lens,
                              void* stream, float* out_logits) {
  if (!h || !tokens || !positions || !seq_lens || !out_logits) return MK_ERR_INVALID_ARG;
  mk::Params p = h->p;
  p.tokens = tokens;
  p.positions = positions;
  p.seq_lens = seq_lens;
  p.logits = out_logits;
  p.epoch = h->epoch + 1;
  cudaError_t e = mk::launch_step(p, h->n_sm, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  h->epoch = p.epoch;
  return MK_OK;
}

namespace {

// Greedy loop: copy the first tokens and the lengths, clear the arg-max words.
__global__ void greedy_init(const int32_t* tok0, const int32_t* len0, int B, int32_t* tok, int32_t* len,
                            unsigned long long* amax) {
  const int b = threadIdx.x;
  if (b < B) {
    tok[b] = tok0[b];
    len[b] = len0[b];
    amax[b] = 0ull;
  }
}

// After a step: the arg-max token (the key's low word holds ~token) becomes the
// next step's input and output, every sequence moves one position on.  A step
// that did no work (a sticky device status) leaves the key at 0: token -1.
__global__ void greedy_advance(int B, int32_t* tok, int32_t* len, unsigned long long* amax, int32_t* out_tok) {
  const int b = threadIdx.x;
  if (b < B) {
    const int token = (int)(0xFFFFFFFFu - (uint32_t)(amax[b] & 0xFFFFFFFFull));
    out_tok[b] = token;
    tok[b] = token;
    len[b] += 1;
    amax[b] = 0ull;
  }
}

}  // namespace

extern "C" int mk_decode_greedy(mk_handle* h, int n_steps, const int32_t* tokens, const int32_t* seq_lens,
                                void* stream, int32_t* out_tokens, float* out_logits) {
  if (!h || n_steps < 0 || !tokens || !seq_lens || (n_steps > 0 && !out_tokens)) return MK_ERR_INVALID_ARG;
  if (n_steps == 0) return MK_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const int B = h->d.batch;
  greedy_init<<<1, 32, 0, st>>>(tokens, seq_lens, B, h->loop_tok, h->loop_len, h->amax);
  if (cudaGetLastError() != cudaSuccess) return MK_ERR_CUDA;
  for (int t = 0; t < n_steps; ++t) {
    mk::Params p = h->p;
    p.tokens = h->loop_tok;
    p.positions = h->loop_len;
    p.seq_lens = h->loop_len;
    p.logits = (t == n_steps - 1 && out_logits) ? out_logits : h->loop_logits;
    p.argmax = h->amax;
    p.epoch = h->epoch + 1;
    if (mk::launch_step(p, h->n_sm, st) != cudaSuccess) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
    h->epoch = p.epoch;
    greedy_advance<<<1, 32, 0, st>>>(B, h->loop_tok, h->loop_len, h->amax, out_tokens + (size_t)t * B);
    if (cudaGetLastError() != cudaSuccess) return MK_ERR_CUDA;
  }
  return MK_OK;
}

extern "C" int mk_get_status(mk_handle* h, void* stream) {
  if (!h) return MK_ERR_INVALID_ARG;
  int st[4] = {0, 0, 0, 0};
  if (cudaMemcpyAsync(st, h->p.status, sizeof(st), cudaMemcpyDeviceToHost, (cudaStream_t)stream) != cudaSuccess ||
      cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
    return MK_ERR_CUDA;
  if (st[0] != 0) {
    // the abandoned step left counters part-way: start again from epoch 0
    if (cudaMemsetAsync(h->p.counters, 0, sizeof(uint32_t) * h->n_counters, (cudaStream_t)stream) != cudaSuccess ||
        cudaMemsetAsync(h->p.tickets, 0, sizeof(uint32_t) * h->n_tickets, (cudaStream_t)stream) != cudaSuccess ||
        cudaMemsetAsync(h->p.status, 0, sizeof(int) * 4, (cudaStream_t)stream) != cudaSuccess ||
        cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
      return MK_ERR_CUDA;
    h->epoch = 0;
  }
  return st[0];
}

extern "C" int mk_destroy(mk_handle* h) {
  if (!h) return MK_OK;
  cudaError_t e = cudaFree(h->region);
  delete h;
  return e == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}

extern "C" size_t mk_state_bytes(const mk_handle* h, int which) {
  if (!h) return 0;
  const mk_model_desc& d = h->d;
  switch (which) {
    case MK_STATE_HIDDEN: return sizeof(float) * (size_t)(2 * d.n_layers + 1) * d.batch * d.hidden;
    case MK_STATE_ROUTER: return sizeof(float) * (size_t)d.n_layers * d.batch * d.n_experts;
    case MK_STATE_SELECTION: return d.n_experts ? sizeof(int32_t) * (size_t)d.n_layers * d.batch * d.top_k : 0;
    case MK_STATE_SEL_WEIGHT: return d.n_experts ? sizeof(float) * (size_t)d.n_layers * d.batch * d.top_k : 0;
    case MK_STATE_EXPERT_COUNT: return d.n_experts ? sizeof(int32_t) * (size_t)d.n_layers : 0;
    case MK_STATE_TRACE: return sizeof(uint64_t) * mk::kTraceStamps * h->n_instr;
    case MK_STATE_COUNTERS: return sizeof(uint32_t) * (size_t)h->n_counters;
    default: return 0;
  }
}

extern "C" int mk_read_state(mk_handle* h, int which, void* dst, size_t bytes, void* stream) {
  if (!h || !dst) return MK_ERR_INVALID_ARG;
  const size_t need = mk_state_bytes(h, which);
  if (need == 0) return MK_ERR_INVALID_ARG;
  if (bytes < need) return MK_ERR_INVALID_ARG;
  const void* src = nullptr;
  if (which == MK_STATE_HIDDEN) src = h->p.xres;
  if (which == MK_STATE_TRACE) src = h->p.trace;
  if (which == MK_STATE_ROUTER) src = h->p.moe_router;
  if (which == MK_STATE_SELECTION) src = h->p.moe_sel;
  if (which == MK_STATE_SEL_WEIGHT) src = h->p.moe_selw;
  if (which == MK_STATE_EXPERT_COUNT) src = h->p.moe_count;
  if (which == MK_STATE_COUNTERS) src = h->p.counters;
  if (cudaMemcpyAsync(dst, src, need, cudaMemcpyDefault, (cudaStream_t)stream) != cudaSuccess) return MK_ERR_CUDA;
  return MK_OK;
}
