// mk_decode_step_noalloc: the decode step for callers that may not allocate
// device memory.
//
// Some callers cannot call cudaMalloc at the point where they decode: a plugin
// running inside another engine's enqueue call, where that engine owns every
// device byte and forbids allocations of its own; code on a real-time path
// that must not block on the allocator; or a process whose memory budget is
// fully reserved up front.  For them this entry point runs the same
// persistent kernel as mk_decode_step, but every byte of library state
// (instruction lists, dependency counters, activation scratch, RoPE table,
// the batch > 1 kernel's TMA tensor maps)
// lives in one file-scope static device array of kStaticScratchBytes (8 MiB).
// Every GPU that loads this library holds that array until the process exits.
//
// The array's host-side name is only a stand-in: its device address is taken
// with cudaGetSymbolAddress once per device (with that device current), on the
// first call made on that device, and passed to the kernel.
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "mk_device.h"
#include "mk_internal.h"

extern "C" int mk_plan_create(const mk_model_desc*, int, mk_plan**);
extern "C" int mk_plan_n_instrs(const mk_plan*);
extern "C" int mk_plan_copy(const mk_plan*, mk_instr*, int32_t*);
extern "C" int mk_plan_n_counters(const mk_plan*);
extern "C" int mk_plan_attn_chunk(const mk_plan*, int32_t*, int32_t*);
extern "C" int mk_plan_destroy(mk_plan*);

namespace mk {
int validate_desc(const mk_model_desc* d);
}

namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;
constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

static __device__ __align__(256) unsigned char g_mk_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of the array, per device
bool g_ready[kMaxDevices];

// Once per device: resolve the array's device address and prepare the kernel.
int device_setup(int dev, void** addr) {
  if (dev < 0 || dev >= kMaxDevices) return MK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_ready[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mk_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
    if (mk::kernel_prepare() != cudaSuccess) return MK_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_ready[dev] = true;
  }
  *addr = g_scratch_addr[dev];
  return MK_OK;
}

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

extern "C" int mk_decode_step_noalloc(const mk_model_desc* desc, const mk_weights* w, const mk_kv* kv,
                                      const int32_t* tokens, const int32_t* positions, const int32_t* seq_lens,
                                      void* stream, float* out_logits) {
  if (!desc || !w || !kv || !w->layers || !tokens || !positions || !seq_lens || !out_logits)
    return MK_ERR_INVALID_ARG;
  int rc = mk::validate_desc(desc);
  if (rc) return rc;
  const mk_model_desc& d = *desc;
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

  int dev = 0, n_sm = 0, coop = 0, smem_optin = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MK_ERR_CUDA;
  void* scratch = nullptr;
  rc = device_setup(dev, &scratch);
  if (rc) return rc;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
      mk::kernel_occupancy(&per_sm, mk::batched(d)) != cudaSuccess)
    return MK_ERR_CUDA;
  if (!coop || (size_t)smem_optin < mk::kernel_smem_bytes(mk::batched(d)) || per_sm < 1) return MK_ERR_UNSUPPORTED;

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

  const int L = d.n_layers, B = d.batch, H = d.hidden, hd = d.head_dim, nq = d.n_q_heads, nkv = d.n_kv_heads;
  const size_t qd = (size_t)nq * hd, kvd = (size_t)nkv * hd;
  // Layout inside the static array.  The first block (counters, tickets,
  // status) must start every call at zero; everything else is overwritten.
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += round256(bytes);
    return o;
  };
  const size_t o_cnt = take(sizeof(uint32_t) * (size_t)n_cnt);
  const int group = nq / nkv;
  const size_t o_tk = take(sizeof(uint32_t) * (size_t)L * B * nkv * (group / mk::attn_heads_per_instr(group)));
  const size_t o_st = take(sizeof(int) * 4);
  const size_t zero_bytes = off;
  const size_t o_xres = take(sizeof(float) * (size_t)(2 * L + 1) * B * H);
  const size_t o_qkv = take(sizeof(float) * (size_t)B * (qd + 2 * kvd));
  const size_t o_attn = take(sizeof(float) * (size_t)B * qd);
  const size_t o_act = take(sizeof(float) * (size_t)B * (d.n_experts ? 1 : d.ffn_dim));
  const int E = d.n_experts, K = d.top_k;
  const size_t o_mr = E ? take(sizeof(float) * (size_t)L * B * E) : 0;
  const size_t o_ms = E ? take(sizeof(int32_t) * (size_t)L * B * K) : 0;
  const size_t o_mw = E ? take(sizeof(float) * (size_t)L * B * K) : 0;
  const size_t o_mc = E ? take(sizeof(int32_t) * (size_t)L) : 0;
  const size_t o_ma = E ? take(sizeof(uint16_t) * (size_t)mk::moe_slots(E, B, K) * B * d.expert_ffn_dim) : 0;
  const size_t o_abf = mk::batched(d) ? take(sizeof(uint16_t) * (size_t)B * qd) : 0;
  const size_t o_xbf = mk::batched(d) && !E ? take(sizeof(uint16_t) * (size_t)B * d.ffn_dim) : 0;
  const size_t o_po = take(sizeof(float) * (size_t)B * nq * n_chunks * hd);
  const size_t o_pml = take(sizeof(float) * (size_t)B * nq * n_chunks * 2);
  const size_t o_ins = take(sizeof(mk_instr) * instrs.size());
  const size_t o_off = take(sizeof(int32_t) * offsets.size());
  const size_t o_lay = take(sizeof(mk::LayerPtrs) * (size_t)L);
  const size_t o_rope = take(sizeof(float2) * (size_t)d.max_ctx * (hd / 2));
  const size_t n_tmaps = (size_t)mk::kTmapsPerLayer * L + 3;  // KV caches always; weights on the tensor-core kernel
  const size_t o_tmap = n_tmaps ? take(128 * n_tmaps) : 0;
  const size_t n_tb1 = mk::batched(d) ? 0 : mk::n_tmaps_b1(d);  // the batch-1 kernel's weight maps
  const size_t o_tb1 = n_tb1 ? take(128 * n_tb1) : 0;
  if (off > kStaticScratchBytes) return MK_ERR_UNSUPPORTED;  // model needs more than the 8 MiB array
  std::vector<uint8_t> tmaps(128 * n_tmaps), tb1(128 * n_tb1);
  cudaError_t te = n_tmaps ? mk::encode_tmaps(d, *w, *kv, tmaps.data()) : cudaSuccess;
  if (te == cudaSuccess && n_tb1) te = mk::encode_tmaps_b1(d, *w, tb1.data());
  if (te != cudaSuccess) return te == cudaErrorInvalidValue ? MK_ERR_UNSUPPORTED : MK_ERR_CUDA;

  std::vector<mk::LayerPtrs> lp(L);
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights& s = w->layers[l];
    lp[l] = mk::LayerPtrs{(const uint16_t*)s.attn_norm, (const uint16_t*)s.wq,     (const uint16_t*)s.wk,
                          (const uint16_t*)s.wv,        (const uint16_t*)s.q_norm, (const uint16_t*)s.k_norm,
                          (const uint16_t*)s.wo,        (const uint16_t*)s.mlp_norm, (const uint16_t*)s.w_gate,
                          (const uint16_t*)s.w_up,      (const uint16_t*)s.w_down, (const uint16_t*)s.router};
  }
  std::vector<float2> rope((size_t)d.max_ctx * (hd / 2));
  for (int pos = 0; pos < d.max_ctx; ++pos)
    for (int i = 0; i < hd / 2; ++i) {
      const double ang = (double)pos * pow((double)d.rope_theta, -2.0 * i / hd);
      rope[(size_t)pos * (hd / 2) + i] = make_float2((float)cos(ang), (float)sin(ang));
    }

  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  // Pageable host sources: each copy has read its source when the call returns.
  if (cudaMemsetAsync(base, 0, zero_bytes, s) != cudaSuccess ||
      cudaMemcpyAsync(base + o_ins, instrs.data(), sizeof(mk_instr) * instrs.size(), cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(base + o_off, offsets.data(), sizeof(int32_t) * offsets.size(), cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(base + o_lay, lp.data(), sizeof(mk::LayerPtrs) * L, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(base + o_rope, rope.data(), sizeof(float2) * rope.size(), cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      (n_tmaps && cudaMemcpyAsync(base + o_tmap, tmaps.data(), tmaps.size(), cudaMemcpyHostToDevice, s) != cudaSuccess) ||
      (n_tb1 && cudaMemcpyAsync(base + o_tb1, tb1.data(), tb1.size(), cudaMemcpyHostToDevice, s) != cudaSuccess))
    return MK_ERR_CUDA;

  mk::Params p;
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
  p.tokens = tokens;
  p.positions = positions;
  p.seq_lens = seq_lens;
  p.logits = out_logits;
  p.epoch = 1;  // counters were just cleared
  if (mk::launch_step(p, n_sm, s) != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  // Report the device-side status of this step (range error, wait timeout).
  int st = 0;
  if (cudaMemcpyAsync(&st, p.status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MK_ERR_CUDA;
  return st;
}
