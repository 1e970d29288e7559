// The persistent decode-step kernel for sm_100a.
//
// One CTA per SM, launched cooperatively so that every CTA is resident.  Each
// CTA walks its own instruction list (built by mk_plan.cpp) with two roles:
//
//  * warp 8, the producer: streams the bytes every instruction reads from
//    HBM and never changes during a step -- weight rows and the KV-cache
//    positions cached by earlier steps -- into a 6-slot x 32 KB shared-memory
//    ring with 1-D bulk copies (cp.async.bulk, completion on an mbarrier,
//    L2 evict-first).  It runs ahead of the compute across instruction and
//    layer boundaries, so weight streaming continues while the consumers wait
//    on a dependency.
//  * warps 0-7, the consumers: wait on the dependency counter of each
//    instruction (bounded spin on an acquire load), compute from the ring
//    (GEMV with a fused RMSNorm prologue and residual / SwiGLU epilogue,
//    split-K attention with an online softmax), write fp32 activations with
//    generic stores, then bump the instruction's counter with a release add.
//
// ForgeMegakernel (arXiv 2609.12379, abstract) gives the properties followed:
// a per-SM instruction stream and dependency counters replacing global
// synchronisation; the page names no data layout, tile shape or instruction
// format, so those below are this library's own.
//
// Failure handling: every wait is bounded by Params::timeout_ns.  A CTA that
// gives up records MK_ERR_DEVICE_TIMEOUT in the status word and every other
// CTA leaves at its next counter wait; the producer waits for its own copies
// in flight before leaving.  Nothing traps.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mk_device.h"

namespace mk {

// ---------------------------------------------------------------------------
// shared memory layout
// ---------------------------------------------------------------------------
struct Ctl {
  unsigned long long full[kStages];
  unsigned long long empty[kStages];
  int dead;       // this CTA gives up: every wait returns at once
  int waiting;    // the consumers are blocked on a dependency counter
  int last;       // attention: this CTA merges (broadcast)
  int flag;       // generic broadcast
  int32_t slen[kMaxBatch], spos[kMaxBatch];  // this step's seq_lens and positions (read once per step)
  uint32_t xtag;  // batch-1 GEMV: which input piece the reduction buffer holds (0: none)
  float xss;      // and, for a norm-fused op, the sum of squares of its input
  float b1red[kB1MaxLines * 4];  // batch-1 GEMV: per-warp sums of lines split over chunks
  // batch-1 GEMV, the producer's current instruction: its TMA boxes for one
  // chunk (tensor map, row, shared-memory offset within the chunk's lines)
  struct B1Box {
    const uint8_t* map;
    int row;
    uint32_t off;
  } b1box[kB1MaxLines];
  int b1nbox;
  float sred[kConsumerWarps * 2];
  alignas(16) float qs[kMaxGroup * kMaxHeadDim];
  float aml[kConsumerWarps * kMaxGroup * 2];  // attention: per-warp (m, l) of every head
  alignas(16) uint16_t knew[kMaxHeadDim];     // the new token's K/V rows (bf16, as appended)
  alignas(16) uint16_t vnew[kMaxHeadDim];
  AttnSched psched;  // the producer's attention schedule of its current slot
  // MoE: the current layer's routing.  The consumers compute it; the
  // producer, which cannot stream expert weights before it exists, waits for
  // moe_pub == layer + 1.
  unsigned long long amax[kMaxBatch];  // greedy decoding: an LM-head instruction's arg-max per sequence
  int moe_pub;
  int moe_count;                       // distinct picked experts (slots)
  int16_t moe_uniq[kMaxSel];           // expert of each slot, ascending
  uint32_t moe_mask[kMaxExperts / 32];
  float moe_tw[kMaxSel][kMaxBatch];    // routing weight of (slot, sequence); 0 if not picked
};

// Shared memory: the ring of weight / KV stages (slots 1024-byte aligned, as
// the swizzled TMA boxes of the batched GEMV need), the reduction buffer, Ctl.
template <bool BATCHED>
struct Smem {
  static constexpr int kNst = BATCHED ? kStagesBatched : kStages;
  static constexpr size_t kSlot = (size_t)kStageBytes;
  static_assert(2 * kBBoxBytes == kStageBytes, "a batched GEMV stage is two boxes");
  static constexpr size_t kRing = (size_t)kNst * kSlot;
  // the reduction buffer doubles as the GEMV input buffer (never both at once): the
  // tensor-core kernel's input ring, the batch-1 kernel's input piece
  static constexpr size_t kXs = BATCHED ? (size_t)kXsSlots * kMaxBatch * kXsPitchBytes
                                        : (size_t)kB1XPieceFloats * sizeof(float);
  static constexpr size_t kRed = (size_t)kRedFloats * sizeof(float) > kXs ? (size_t)kRedFloats * sizeof(float) : kXs;
  static constexpr size_t kTotal = kRing + kRed + sizeof(Ctl);
  static_assert(kNst <= kStages, "Ctl holds kStages barrier pairs");
  static_assert(kTotal <= 227 * 1024, "dynamic shared memory of one CTA");
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(unsigned long long* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// 16 bytes global -> shared, asynchronous, cached in L2 only (the source may
// have been written by another SM during this kernel).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// all but the newest N committed groups of this thread have landed
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One box of a 3-D tensor map (coordinates c0, c1, c2) into shared memory,
// completing on `bar`.
__device__ __forceinline__ void tma_box3(void* dst, const void* map, int c0, int c1, int c2, unsigned long long* bar,
                                         uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

// One box of a 2-D tensor map (column c0, row c1) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_box2(void* dst, const void* map, int c0, int c1, unsigned long long* bar,
                                         uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, unsigned long long* bar,
                                         uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int ld_relaxed_i32(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Named barrier 1 over the 256 consumer threads, OR-reducing a predicate.
__device__ __forceinline__ bool consumer_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Reduce R independent per-lane values over the 32 lanes of a warp with
// R - 1 + 5 - log2(R) shuffles: each butterfly level halves the number of
// values a lane carries (the lane keeps one half and receives its partner's
// copy of that half), then plain xor levels finish the sum.  Afterwards lane l
// holds the total of value index row_of_lane<R>(l) (lanes sharing the top
// log2(R) bits hold the same total).
__host__ __device__ constexpr int ilog2c(int x) { return x <= 1 ? 0 : 1 + ilog2c(x / 2); }

// The same over groups of LPP consecutive lanes (R <= LPP): afterwards lane l
// holds the group total of value index (l % LPP) >> (log2 LPP - log2 R).
template <int R, int LPP>
__device__ __forceinline__ float group_reduce_multi(float (&v)[R], int lane) {
  constexpr int LOG = ilog2c(R);
#pragma unroll
  for (int lvl = 0; lvl < LOG; ++lvl) {
    const int off = (LPP / 2) >> lvl;
    const int half = R >> (lvl + 1);
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < (R >> 1); ++k) {
      if (k < half) {
        const float send = up ? v[k] : v[k + half];
        const float keep = up ? v[k + half] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
  }
  float s = v[0];
#pragma unroll
  for (int off = (LPP / 2) >> LOG; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  return s;
}

template <int R>
__device__ __forceinline__ float warp_reduce_multi(float (&v)[R], int lane) {
  return group_reduce_multi<R, 32>(v, lane);
}

template <int R>
__device__ __forceinline__ int row_of_lane(int lane) {
  constexpr int LOG = R >= 16 ? 4 : R >= 8 ? 3 : R >= 4 ? 2 : R >= 2 ? 1 : 0;
  int r = 0;
#pragma unroll
  for (int lvl = 0; lvl < LOG; ++lvl) r |= ((lane >> (4 - lvl)) & 1) << (LOG - 1 - lvl);
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

__device__ __forceinline__ void unpack8(const uint4 w, float f[8]) {
  f[0] = bf16_lo(w.x); f[1] = bf16_hi(w.x);
  f[2] = bf16_lo(w.y); f[3] = bf16_hi(w.y);
  f[4] = bf16_lo(w.z); f[5] = bf16_hi(w.z);
  f[6] = bf16_lo(w.w); f[7] = bf16_hi(w.w);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits_fwd(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

// 8-term dot product in two interleaved FMA chains (shorter dependency chain).
__device__ __forceinline__ float dot8(const uint4 w, const float x[8], float acc) {
  float b = 0.f;
  acc = fmaf(bf16_lo(w.x), x[0], acc);
  b = fmaf(bf16_hi(w.x), x[1], b);
  acc = fmaf(bf16_lo(w.y), x[2], acc);
  b = fmaf(bf16_hi(w.y), x[3], b);
  acc = fmaf(bf16_lo(w.z), x[4], acc);
  b = fmaf(bf16_hi(w.z), x[5], b);
  acc = fmaf(bf16_lo(w.w), x[6], acc);
  b = fmaf(bf16_hi(w.w), x[7], b);
  return acc + b;
}

// Packed fp32 pairs (sm_100 fma.rn.f32x2: two IEEE fp32 FMAs per instruction).
__device__ __forceinline__ unsigned long long pack2(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ float sum2(unsigned long long a) {
  float x, y;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(a));
  return x + y;
}

// 8 bf16 weights times 8 packed fp32 inputs, accumulated as fp32 pairs.
__device__ __forceinline__ unsigned long long dot8x2(const uint4 w, const unsigned long long xp[4],
                                                     unsigned long long acc) {
  acc = ffma2(pack2(bf16_lo(w.x), bf16_hi(w.x)), xp[0], acc);
  acc = ffma2(pack2(bf16_lo(w.y), bf16_hi(w.y)), xp[1], acc);
  acc = ffma2(pack2(bf16_lo(w.z), bf16_hi(w.z)), xp[2], acc);
  acc = ffma2(pack2(bf16_lo(w.w), bf16_hi(w.w)), xp[3], acc);
  return acc;
}

// D += A(16x16, row) * B(16x8, col), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Greedy decoding: a logit and its token packed so that the unsigned maximum
// is the largest logit and, among equal logits, the lowest token id.
__device__ __forceinline__ unsigned long long argmax_key(float y, int token) {
  uint32_t u = __float_as_uint(y);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // order-preserving map of the float
  return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)token);
}

// Two fp32 values rounded to nearest-even bf16, `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 16-byte loads from shared memory at a 32-bit shared address.
__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
// The same, predicated: zeros where `pred` is 0 (no branch around the load).
__device__ __forceinline__ uint4 lds_u4_if(uint32_t a, uint32_t pred) {
  uint4 v;
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %5, 0;\n\t"
      "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
      "@p ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "r"(a), "r"(pred));
  return v;
}
__device__ __forceinline__ float4 lds_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}

// Four 8x8 b16 matrices from shared memory, transposed on the way: lane
// (g, c) receives elements (2c, g) and (2c + 1, g) of every stored matrix.
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t a[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(saddr));
}

// Transpose of an 8x8 b16 matrix held one element pair per lane (lane (g, c)
// holds row g, columns 2c and 2c + 1) into the same layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Four 8x8 b16 matrices from shared memory; lane l supplies the address of
// row (l & 7) of matrix (l >> 3) and receives element pair (l >> 2, 2 * (l & 3))
// of every matrix: exactly an m16n8k16 A fragment when the matrices are
// (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15).
__device__ __forceinline__ void ldmatrix_x4(uint32_t a[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(saddr));
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ void set_status(const Params& p, int code, int detail) {
  if (atomicCAS(p.status, 0, code) == 0) {
    p.status[1] = detail;
    p.status[2] = blockIdx.x;
  }
}

// ---------------------------------------------------------------------------
// Instruction geometry (identical on the producer and consumer side)
// ---------------------------------------------------------------------------
// A GEMV instruction covers rows [r0, r1) of its op's row space.  For QKV that
// space is wq | wk | wv concatenated, so an instruction may span up to three
// matrices ("segments").  Fields are named (not arrays) so that the geometry
// stays in registers.
struct Gemv {
  int K, r0, r1;
  bool gated;  // gate/up: every row is a pair of lines, gate then up
  // batch > 1 (tensor cores): bnch chunks of kBChunk columns, bnt tiles of
  // btile_rows() output rows
  int bnch, bnt;
  // batch 1 (row-stationary tiles): lines of the instruction, chunks of
  // kB1Chunk columns, chunks per stage, stages; per segment its first box map
  // (the others follow it), first row within its matrix, rows and first line
  // within a stage
  int lines, nch, ncs, nst, nseg;
  // gate/up of more than kB1MaxLines / 2 neurons: a stage holds one group (the
  // gate rows or the up rows) of one chunk, gate then up for every chunk
  bool split;
  const uint8_t *bm0, *bm1, *bm2;
  int brow0, brow1, brow2, bn0, bn1, bn2, bl0, bl1, bl2;
  __device__ __forceinline__ int seg_rows(int s) const { return s == 0 ? bn0 : (s == 1 ? bn1 : bn2); }
  __device__ __forceinline__ int seg_row(int s) const { return s == 0 ? brow0 : (s == 1 ? brow1 : brow2); }
  __device__ __forceinline__ int seg_line(int s) const { return s == 0 ? bl0 : (s == 1 ? bl1 : bl2); }
  __device__ __forceinline__ const uint8_t* seg_map(int s) const { return s == 0 ? bm0 : (s == 1 ? bm1 : bm2); }
};

// Batch-1 box maps of matrix `mat` (0..6: wq wk wv wo w_gate w_up w_down) of
// a layer: kB1BoxHeights maps, of 64, 32, 16, 8, 4, 2 and 1 rows.
__device__ __forceinline__ const uint8_t* b1_map(const Params& p, int layer, int mat) {
  return p.tmaps_b1 + ((size_t)layer * kB1MapsPerLayer + kB1BoxHeights * mat) * 128;
}

__device__ __forceinline__ Gemv gemv_geo(const Params& p, const mk_instr& in, int op, int layer) {
  Gemv g;
  g.r0 = in.a;
  g.r1 = in.b;
  g.gated = op == OP_GATEUP;
  const int R = g.r1 - g.r0;
  g.nseg = 1;
  g.bn0 = R;
  g.bn1 = g.bn2 = 0;
  g.brow0 = g.r0;
  g.brow1 = g.brow2 = 0;
  g.bl0 = 0;
  g.bl1 = g.bl2 = 0;
  g.bm0 = g.bm1 = g.bm2 = nullptr;
  if (op == OP_LMHEAD) {
    g.K = p.H;
    if (!p.tc) {
      g.bm0 = p.tmaps_b1 + (size_t)p.L * kB1MapsPerLayer * 128;
    }
  } else {
    switch (op) {
      case OP_QKV: {
        g.K = p.H;
        if (!p.tc) {
          const int qd = p.nq * p.hd, kvd = p.nkv * p.hd;
          g.nseg = 0;
#pragma unroll
          for (int m = 0; m < 3; ++m) {
            const int base = m == 0 ? 0 : (m == 1 ? qd : qd + kvd);
            const int end = m == 0 ? qd : (m == 1 ? qd + kvd : qd + 2 * kvd);
            const int a = max(g.r0, base), b = min(g.r1, end);
            if (a < b) {
              const uint8_t* map = b1_map(p, layer, m);
              if (g.nseg == 0) { g.bm0 = map; g.brow0 = a - base; g.bn0 = b - a; g.bl0 = a - g.r0; }
              else if (g.nseg == 1) { g.bm1 = map; g.brow1 = a - base; g.bn1 = b - a; g.bl1 = a - g.r0; }
              else { g.bm2 = map; g.brow2 = a - base; g.bn2 = b - a; g.bl2 = a - g.r0; }
              ++g.nseg;
            }
          }
        }
        break;
      }
      case OP_OPROJ:
        g.K = p.nq * p.hd;
        if (!p.tc) g.bm0 = b1_map(p, layer, 3);
        break;
      case OP_GATEUP:
        g.K = p.H;
        if (!p.tc) {  // gate rows, then the same rows of up
          g.nseg = 2;
          g.bm0 = b1_map(p, layer, 4);
          g.bm1 = b1_map(p, layer, 5);
          g.brow1 = g.r0;
          g.bn1 = R;
          g.bl1 = R;
        }
        break;
      case OP_ROUTER:
        g.K = p.H;
        break;
      case OP_EXP_DOWN:  // rows of every picked expert's down matrix (tensor maps)
        g.K = p.Ie;
        break;
      default:  // OP_DOWN
        g.K = p.I;
        if (!p.tc) g.bm0 = b1_map(p, layer, 6);
        break;
    }
  }
  g.lines = R * (g.gated ? 2 : 1);
  g.nch = (g.K + kB1Chunk - 1) / kB1Chunk;
  g.ncs = b1_chunks_per_stage(g.lines);
  g.nst = (g.nch + g.ncs - 1) / g.ncs;
  g.split = !p.tc && g.gated && g.lines > kB1MaxLines;
  if (g.split) {  // both groups start at line 0 of their stages
    g.bl1 = 0;
    g.lines = R;
    g.ncs = 1;
    g.nst = 2 * g.nch;
  }
  if (p.tc) {
    const int tr = btile_rows(g.gated);
    g.bnch = (g.K + kBChunk - 1) / kBChunk;
    g.bnt = (R + tr - 1) / tr;
  }
  return g;
}

// MoE down: its K runs over the picked experts one after another, each in
// chunks of kBChunk of its Ie columns.
__device__ __forceinline__ int moe_down_chunks(const Params& p) { return (p.Ie + kBChunk - 1) / kBChunk; }

// MoE gate/up: the piece of an expert slot instruction that starts at unit g
// (units are (slot, 8-neuron tile), slot-major) and ends by g1, at most
// kBatchedMaxRowsGated rows.  Geometry in the stacked [E * Ie] row space.
__device__ __forceinline__ Gemv moe_gate_piece(const Params& p, const Ctl* ctl, int layer, int64_t g, int64_t g1,
                                               int* slot) {
  const int nte = p.Ie / 8;
  const int s = (int)(g / nte), t0 = (int)(g % nte);
  const int64_t left = g1 - g < (int64_t)(kBatchedMaxRowsGated / 8) ? g1 - g : (int64_t)(kBatchedMaxRowsGated / 8);
  const int t1 = (int)(nte - t0 < left ? nte : t0 + left);
  const int e = ctl->moe_uniq[s];
  Gemv gm;
  gm.K = p.H;
  gm.r0 = e * p.Ie + t0 * 8;
  gm.r1 = e * p.Ie + t1 * 8;
  gm.gated = true;
  gm.split = false;
  gm.bnch = (p.H + kBChunk - 1) / kBChunk;
  gm.bnt = t1 - t0;
  *slot = s;
  return gm;
}

// One attention piece: units [ua, ub) of row (b, kvh, hg), i.e. positions
// [p0, min(ub * unit, S + 1)); the cached ones [p0, p0 + n_cached) stream
// through the ring, the new token (position S) comes from this step's qkv.
struct Attn {
  int b, kvh, hg, S, p0, n_cached, nsub, P;
  int c, npieces;  // index of the piece within its row, pieces of the row
  bool active, owns_new;
};

// Row (of head_dim elements) of (layer, sequence b, KV head, position) in
// the K or V cache: contiguous [L][B][nkv][T], or paged [L][n_pages][nkv][page]
// through the block table.
__device__ __forceinline__ int64_t kv_row(const Params& p, int layer, int b, int kvh, int pos) {
  if (p.bt) {
    const int page = __ldg(p.bt + (size_t)b * p.bt_stride + pos / p.page);
    return (((int64_t)layer * p.n_pages + page) * p.nkv + kvh) * p.page + pos % p.page;
  }
  return (((int64_t)layer * p.B + b) * p.nkv + kvh) * p.T + pos;
}

__device__ __forceinline__ Attn attn_geo(const Params& p, const Ctl* ctl, const AttnPiece& pc, int layer, int head_dim) {
  Attn a;
  const int group = p.nq / p.nkv, nhg = group / attn_heads_per_instr(group);
  a.b = pc.b;
  a.kvh = pc.row / nhg;
  a.hg = pc.row % nhg;
  a.S = ctl->slen[a.b];
  a.p0 = pc.ua * p.chunk;
  const int p1 = pc.ub * p.chunk;
  a.active = true;
  a.owns_new = a.S < p1;
  a.n_cached = max(0, min(p1, a.S) - a.p0);
  a.P = attn_stage_positions(head_dim);
  a.nsub = (a.n_cached + a.P - 1) / a.P;
  a.c = pc.slot_in_row;
  a.npieces = pc.n_pieces;
  return a;
}

__device__ __forceinline__ void attn_sched(const Params& p, const Ctl* ctl, const mk_instr& in, AttnSched& sc) {
  const int group = p.nq / p.nkv;
  attn_sched_init(sc, ctl->slen, p.B, p.nkv * (group / attn_heads_per_instr(group)), p.chunk, in.b);
}

// ---------------------------------------------------------------------------
// Producer warp (lane 0 issues everything)
// ---------------------------------------------------------------------------

// Walks the stages of an SM's instruction list in order.  A GEMV stage is R
// rows (one column slice) of one segment, plus the same rows of the up matrix
// for gate/up; an attention stage is up to P cached positions of K or of V.
struct Cursor {
  const Params* pp;  // pointer (not reference) so that cursors can be assigned
  const mk_instr* list;
  int n;
  int i;  // instruction index; >= n when every stage has been walked
  int op, layer;
  Gemv g;
  int kc, sg, rr;  // GEMV: slice (batched: chunk), segment (batched: tile), first row within the segment
  Attn a;
  int sub, kv;     // attention: stage within the piece, K (0) or V (1)
  AttnSched* sc;   // attention: this step's schedule (shared memory), slot aslot's units [ag, ag1)
  int64_t ag, ag1;
  int aslot, pieceu;  // slot, units of the current piece
  const Ctl* ctl;     // MoE: the layer's routing
  bool pending;       // an expert instruction waits for its layer's routing
  int eslot;          // MoE gate/up: expert slot of the current piece (units [ag, ag1) as above)

  __device__ Cursor(const Params& prm, const mk_instr* l, int nn, AttnSched* sched, const Ctl* c)
      : pp(&prm), list(l), n(nn), i(0), sc(sched), ctl(c), pending(false) {}

  // Position on the first stage of instruction j or of the next one that has stages.
  __device__ __forceinline__ void seek(int j) {
    for (i = j; i < n; ++i) {
      const mk_instr in = list[i];
      op = op_of(in.op_layer);
      layer = layer_of(in.op_layer);
      if (op == OP_ATTN) {
        attn_sched(*pp, ctl, in, *sc);
        aslot = in.a;
        ag = attn_slot_begin(*sc, aslot);
        ag1 = attn_slot_begin(*sc, aslot + 1);
        sub = kv = 0;
        if (next_piece()) return;
      } else if (op == OP_EXP_GATEUP || op == OP_EXP_DOWN) {
        if (*(const volatile int*)&ctl->moe_pub != layer + 1) {
          pending = true;  // the producer waits, then seeks here again
          return;
        }
        __threadfence_block();
        kc = sg = rr = 0;
        if (op == OP_EXP_DOWN) {
          g = gemv_geo(*pp, in, op, layer);
          g.bnch = ctl->moe_count * moe_down_chunks(*pp);
          if (g.bnch > 0) return;
        } else {
          const int64_t U = (int64_t)ctl->moe_count * (pp->Ie / 8);
          ag = even_begin(U, in.b, in.a);
          ag1 = even_begin(U, in.b, in.a + 1);
          if (next_moe_piece()) return;
        }
      } else if ((op >= OP_QKV && op <= OP_LMHEAD) || op == OP_ROUTER) {
        g = gemv_geo(*pp, in, op, layer);
        kc = sg = rr = 0;
        return;
      }
    }
  }

  // MoE gate/up: the piece of the slot that starts at unit ag, if any.
  __device__ __forceinline__ bool next_moe_piece() {
    if (ag >= ag1) return false;
    g = moe_gate_piece(*pp, ctl, layer, ag, ag1, &eslot);
    kc = sg = rr = 0;
    return true;
  }

  // From unit ag on: the first piece of the slot that has cached positions.
  __device__ __forceinline__ bool next_piece() {
    while (ag < ag1) {
      const AttnPiece pc = attn_piece_at(*sc, ag, aslot);
      a = attn_geo(*pp, ctl, pc, layer, pp->hd);
      pieceu = pc.ub - pc.ua;
      if (a.nsub > 0) return true;
      ag += pieceu;
    }
    return false;
  }

  __device__ __forceinline__ void advance() {
    if (op == OP_ATTN) {
      kv ^= 1;
      if (!kv && ++sub >= a.nsub) {
        sub = 0;
        ag += pieceu;
        if (!next_piece()) seek(i + 1);
      }
      return;
    }
    if (pp->tc) {  // batched GEMV: chunk kc, tile sg within it
      if (++sg >= g.bnt) {
        sg = 0;
        if (++kc >= g.bnch) {
          if (op == OP_EXP_GATEUP) {
            ag += g.bnt;
            if (next_moe_piece()) return;
          }
          seek(i + 1);
        }
      }
      return;
    }
    if (++kc >= g.nst) seek(i + 1);  // batch-1 GEMV: stage kc of the row-stationary tiles
  }

  // Batch-1 GEMV: the TMA boxes of one chunk of every line, into `box` (the
  // same for every chunk but for the column): a segment's rows as boxes of 64,
  // 32, 16, 8, 4, 2 and 1 rows, largest first (single rows only when K is narrower
  // than a chunk, whose boxes are K wide).  Chunk j's line l lands at
  // shared-memory line (j - first chunk of the stage) * lines + l.  Returns
  // the number of boxes; *nb0 = those of the first segment.
  __device__ __forceinline__ int b1_box_list(Ctl::B1Box* box, int* nb0) const {
    const bool wide = g.K >= kB1Chunk;
    int nb = 0;
    *nb0 = 0;
    for (int s2 = 0; s2 < g.nseg; ++s2) {
      if (s2 == 1) *nb0 = nb;
      const uint8_t* map = g.seg_map(s2);
      const int n = g.seg_rows(s2), row = g.seg_row(s2), line = g.seg_line(s2);
      int r = 0;
      for (int m = wide ? 0 : kB1BoxHeights - 1; m < kB1BoxHeights; ++m) {
        const int h = kB1TallestBox >> m;
        for (; r + h <= n; r += h) {
          box[nb].map = map + 128 * m;
          box[nb].row = row + r;
          box[nb].off = (uint32_t)(line + r) * kB1LineBytes;
          ++nb;
        }
      }
    }
    return nb;
  }

  // Batched GEMV stage: f(tensor map, row, column block, shared-memory
  // offset) per TMA box: the two 8-row halves of 16-row tile sg (the second
  // only if the tile has more than 8 rows), or gate over up rows of 8-row tile
  // sg, at column chunk kc.  Returns the stage's bytes.
  template <typename F>
  __device__ __forceinline__ uint32_t boxes(F&& f) const {
    const Params& p = *pp;
    const int kb = kc * (kBChunk / 64);
    if (g.gated) {
      const uint8_t* m = p.tmaps + ((size_t)layer * kTmapsPerLayer + 4) * 128;
      const int row = g.r0 + sg * 8;
      f(m, row, kb, 0u);
      f(m + 128, row, kb, (uint32_t)kBBoxBytes);
      return 2u * kBBoxBytes;
    }
    const int nh = g.r1 - g.r0 - sg * 16 > 8 ? 2 : 1;
    int kbx = kb, rowx = 0;
    if (op == OP_EXP_DOWN) {  // chunk kc = (slot, column chunk of that expert's down rows)
      const int nd = moe_down_chunks(p);
      kbx = (kc % nd) * (kBChunk / 64);
      rowx = ctl->moe_uniq[kc / nd] * p.H;
    }
    for (int h = 0; h < nh; ++h) {
      int row = g.r0 + sg * 16 + h * 8, m;
      if (op == OP_QKV) {
        const int qd = p.nq * p.hd, kvd = p.nkv * p.hd;
        m = row < qd ? 0 : (row < qd + kvd ? 1 : 2);
        row -= m == 0 ? 0 : (m == 1 ? qd : qd + kvd);
      } else {
        m = op == OP_OPROJ ? 3 : (op == OP_ROUTER ? 7 : 6);
      }
      const uint8_t* map = op == OP_LMHEAD ? p.tmaps + (size_t)p.L * kTmapsPerLayer * 128
                                           : p.tmaps + ((size_t)layer * kTmapsPerLayer + m) * 128;
      f(map, row + rowx, kbx, (uint32_t)(h * kBBoxBytes));
    }
    return (uint32_t)nh * kBBoxBytes;
  }

  // Batched attention stage: one box of P positions of the K (kv = 0) or V
  // cache, rows past the chunk's cached positions included (the consumers
  // mask them).
  __device__ __forceinline__ void attn_box(const uint8_t** map, int* row) const {
    const Params& p = *pp;
    *map = p.tmaps + ((size_t)p.L * kTmapsPerLayer + 1 + kv) * 128;
    *row = (int)kv_row(p, layer, a.b, a.kvh, a.p0 + sub * a.P);
  }

  __device__ __forceinline__ uint32_t stage_bytes() const {
    if (op == OP_ATTN)
      return (uint32_t)kStageBytes;  // a TMA box: always a whole stage of positions
    if (pp->tc) return (g.gated || g.r1 - g.r0 - sg * 16 > 8) ? 2u * kBBoxBytes : (uint32_t)kBBoxBytes;
    // batch 1: every line of every chunk of the stage, one box width each
    if (g.split) return (uint32_t)g.lines * (uint32_t)min(g.K, kB1Chunk) * 2u;  // one group of one chunk
    const int j0 = kc * g.ncs, nj = min(g.nch, j0 + g.ncs) - j0;
    return (uint32_t)(g.lines * nj) * (uint32_t)min(g.K, kB1Chunk) * 2u;
  }
};

template <bool BATCHED>
struct Producer {
  static constexpr int NST = Smem<BATCHED>::kNst;
  const Params& p;
  Ctl* ctl;
  uint8_t* ring;
  uint64_t pol;
  uint32_t k = 0;  // stages issued

  __device__ Producer(const Params& pp, Ctl* c, uint8_t* r) : p(pp), ctl(c), ring(r) { pol = evict_first_policy(); }

  // MoE: wait (bounded) until the consumers have put layer `layer`'s routing in place.
  __device__ __forceinline__ bool wait_routing(int layer) {
    const uint64_t t0 = globaltimer();
    uint32_t spins = 0;
    while (*(const volatile int*)&ctl->moe_pub != layer + 1) {
      if (*(volatile int*)&ctl->dead) return false;
      if ((++spins & 63) == 0) {
        if (ld_relaxed_i32(p.status) != 0) return false;
        if (globaltimer() - t0 > p.timeout_ns) {
          set_status(p, MK_ERR_DEVICE_TIMEOUT, -4);
          return false;
        }
      }
    }
    __threadfence_block();
    return true;
  }

  // Claim the next slot (waiting until the consumers released it).
  // on_wait() runs while the ring is full and the consumers wait on a dependency.
  template <typename F>
  __device__ __forceinline__ bool claim(uint8_t** dst, unsigned long long** bar, F&& on_wait) {
    const int slot = k % NST;
    if (k >= (uint32_t)NST) {
      const uint32_t parity = ((k / NST) - 1) & 1;
      if (!mbar_try_wait(&ctl->empty[slot], parity)) {
        const uint64_t t0 = globaltimer();
        uint32_t spins = 0;
        while (!mbar_try_wait(&ctl->empty[slot], parity)) {
          if (*(volatile int*)&ctl->waiting) on_wait();
          if (*(volatile int*)&ctl->dead) return false;
          if ((++spins & 63) == 0) {
            if (ld_relaxed_i32(p.status) != 0) return false;
            if (globaltimer() - t0 > p.timeout_ns) {
              set_status(p, MK_ERR_DEVICE_TIMEOUT, -1);
              return false;
            }
          }
        }
      }
    }
    *dst = ring + (size_t)slot * Smem<BATCHED>::kSlot;
    *bar = &ctl->full[slot];
    return true;
  }

  // After giving up: wait (bounded) for the copies still in flight.
  __device__ __forceinline__ void drain() {
    const uint32_t first = k > (uint32_t)NST ? k - NST : 0;
    for (uint32_t j = first; j < k; ++j) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&ctl->full[j % NST], (j / NST) & 1)) {
        if (globaltimer() - t0 > p.timeout_ns) break;
      }
    }
  }
};

// One thread (lane 0 of the producer warp) issues every copy.
template <bool BATCHED>
__device__ __forceinline__ void run_producer(const Params& p, const mk_instr* list, int n, Ctl* ctl, uint8_t* ring) {
  Producer<BATCHED> pr(p, ctl, ring);
  uint64_t* trace = p.trace ? p.trace + (size_t)p.offsets[blockIdx.x] * kTraceStamps : nullptr;
  Cursor cur(p, list, n, &ctl->psched, ctl);
  cur.seek(0);
  bool ok = true;
  int last = -1;
  while (cur.i < n) {
    if (cur.pending) {  // an expert instruction: its weights follow from the routing
      if (!(ok = pr.wait_routing(cur.layer))) break;
      cur.pending = false;
      cur.seek(cur.i);
      continue;
    }
    if (trace && cur.i != last) {
      const uint64_t now = globaltimer();
      if (last >= 0) trace[last * kTraceStamps + 7] = now;
      for (int j = last + 1; j <= cur.i; ++j) trace[j * kTraceStamps + 3] = now;
      last = cur.i;
    }
    if (!BATCHED) {
      if (cur.op != OP_ATTN) {
        // a batch-1 GEMV instruction: its box list once, then every stage from it
        Ctl::B1Box* box = ctl->b1box;
        int nb0;
        const int nbox = cur.b1_box_list(box, &nb0);
        const int nch = cur.g.nch, ncs = cur.g.ncs, nst = cur.g.nst;
        const uint32_t chunk_stride = (uint32_t)cur.g.lines * kB1LineBytes;
        const uint32_t chunk_bytes = (uint32_t)cur.g.lines * (uint32_t)min(cur.g.K, kB1Chunk) * 2u;
        if (cur.g.split) {
          // two groups: stage 2c holds chunk c of the gate rows, stage 2c + 1 of the up rows
          for (int kc = 0; kc < nst && ok; ++kc) {
            uint8_t* dst;
            unsigned long long* bar;
            if (!(ok = pr.claim(&dst, &bar, [&]() {}))) break;
            mbar_arrive_expect_tx(bar, chunk_bytes);
            const int col = (kc >> 1) * kB1Chunk, b0 = (kc & 1) ? nb0 : 0, b1 = (kc & 1) ? nbox : nb0;
            for (int b = b0; b < b1; ++b) tma_box2(dst + box[b].off, box[b].map, col, box[b].row, bar, pr.pol);
            ++pr.k;
          }
        } else {
          for (int kc = 0; kc < nst && ok; ++kc) {
            uint8_t* dst;
            unsigned long long* bar;
            if (!(ok = pr.claim(&dst, &bar, [&]() {}))) break;
            const int j0 = kc * ncs, nj = min(nch - j0, ncs);
            mbar_arrive_expect_tx(bar, chunk_bytes * (uint32_t)nj);
            for (int jj = 0; jj < nj; ++jj) {
              uint8_t* dj = dst + jj * chunk_stride;
              const int col = (j0 + jj) * kB1Chunk;
              for (int b = 0; b < nbox; ++b) tma_box2(dj + box[b].off, box[b].map, col, box[b].row, bar, pr.pol);
            }
            ++pr.k;
          }
        }
        if (!ok) break;
        cur.seek(cur.i + 1);
        continue;
      }
    }
    uint8_t* dst;
    unsigned long long* bar;
    if (!(ok = pr.claim(&dst, &bar, [&]() {}))) break;
    const uint32_t bytes = cur.stage_bytes();
    mbar_arrive_expect_tx(bar, bytes);
    if (cur.op == OP_ATTN) {
      const uint8_t* map;
      int row;
      cur.attn_box(&map, &row);
      tma_box3(dst, map, 0, row, 0, bar, pr.pol);
    } else {
      cur.boxes([&](const uint8_t* map, int row, int kb, uint32_t off) {
        tma_box3(dst + off, map, 0, row, kb, bar, pr.pol);
      });
    }
    ++pr.k;
    cur.advance();
  }
  if (trace && last >= 0) trace[last * kTraceStamps + 7] = globaltimer();
  if (!ok) {
    ctl->dead = 1;
    pr.drain();
  }
}

// ---------------------------------------------------------------------------
// Consumer warps
// ---------------------------------------------------------------------------
template <bool BATCHED>
struct Consumer {
  static constexpr int NST = Smem<BATCHED>::kNst;
  const Params& p;
  Ctl* ctl;
  uint8_t* ring;
  float* red;
  uint32_t k = 0;  // stages consumed
  uint64_t* tr = nullptr;  // this instruction's trace stamps (thread 0, tracing only)
  const int t = threadIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  __device__ Consumer(const Params& pp, Ctl* c, uint8_t* r, float* rd) : p(pp), ctl(c), ring(r), red(rd) {}

  // Wait until slot k holds its data.  Never changes control flow: on a
  // timeout it marks the CTA dead and returns, and the caller carries on
  // until the next uniform decision point.
  __device__ __forceinline__ const uint8_t* wait_full() { return wait_stage(k); }

  __device__ __forceinline__ const uint8_t* wait_stage(uint32_t kk) {
    const int slot = kk % NST;
    const uint32_t parity = (kk / NST) & 1;
    if (!mbar_try_wait(&ctl->full[slot], parity)) {
      const uint64_t t0 = globaltimer();
      uint32_t spins = 0;
      while (!mbar_try_wait(&ctl->full[slot], parity)) {
        if (*(volatile int*)&ctl->dead) break;
        if ((++spins & 63) == 0 && globaltimer() - t0 > p.timeout_ns) {
          set_status(p, MK_ERR_DEVICE_TIMEOUT, -2);
          ctl->dead = 1;
          break;
        }
      }
    }
    return ring + (size_t)slot * Smem<BATCHED>::kSlot;
  }

  __device__ __forceinline__ void release() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->empty[k % NST]);
    ++k;
  }

  // Dependency wait on `idx` reaching epoch * count.  Uniform result.  An
  // instruction that waits on what the previous wait already saw (the later
  // instructions of an op on this SM) skips the acquire round trip: the data
  // it reads was ordered by that acquire.
  int sat_idx = -1, sat_count = 0;
  __device__ __forceinline__ bool wait_counter(int idx, int count) {
    if (idx >= 0 && idx == sat_idx && count == sat_count) return !consumer_bar_or(*(volatile int*)&ctl->dead != 0);
    sat_idx = idx;
    sat_count = count;
    bool fail = false;
    if (idx >= 0 && t == 0) {
      const uint32_t target = p.epoch * (uint32_t)count;
      const uint32_t* c = p.counters + idx;
      if ((int32_t)(ld_acquire(c) - target) < 0) {
        *(volatile int*)&ctl->waiting = 1;
        const uint64_t t0 = globaltimer();
        while (true) {
          if ((int32_t)(ld_acquire(c) - target) >= 0) break;
          if (ld_relaxed_i32(p.status) != 0 || *(volatile int*)&ctl->dead) {
            fail = true;
            break;
          }
          if (globaltimer() - t0 > p.timeout_ns) {
            set_status(p, MK_ERR_DEVICE_TIMEOUT, idx);
            fail = true;
            break;
          }
        }
        *(volatile int*)&ctl->waiting = 0;
      }
    }
    if (t == 0 && *(volatile int*)&ctl->dead) fail = true;
    return !consumer_bar_or(fail);
  }

  // The named barrier orders every consumer thread's stores of this
  // instruction before thread 0's release reduction; a gpu-scope release is
  // cumulative over what is ordered before it, so an SM that acquires the
  // counter sees all of them.
  __device__ __forceinline__ void signal(int idx) {
    consumer_bar();
    if (t == 0 && idx >= 0) red_release_add(p.counters + idx, 1u);
  }

  // Block-wide sum over the 256 consumer threads (result in every thread).
  __device__ __forceinline__ float block_sum(float v) {
    v = warp_sum(v);
    consumer_bar();
    if (lane == 0) ctl->sred[warp] = v;
    consumer_bar();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) s += ctl->sred[w];
    return s;
  }

  // ---- embedding ------------------------------------------------------------
  __device__ __forceinline__ void embed(const mk_instr& in) {
    for (int b = 0; b < p.B; ++b) {
      const uint16_t* row = p.embed + (size_t)p.tokens[b] * p.H;
      float* x = p.xres + (size_t)b * p.H;
      for (int i = in.a + t; i < in.b; i += kConsumerThreads) x[i] = bf16_bits_to_f32(row[i]);
    }
  }

  // ---- GEMV, batch 1: gate/up of more than 32 neurons ------------------------
  // The instruction's gate rows and its up rows stream as two groups, a stage
  // holding one group's R <= 64 lines of one chunk: chunk c's gate stage, then
  // its up stage.  Warp w owns the neurons w, w + 8, ... (< R); the partial
  // sums of their gate and up lines stay in registers as fp32, each stage's
  // pair of fma chains folded in (16 values per lane, as many registers as the
  // 8 packed pairs of the one-group path), and one 16-value warp reduction
  // ends the instruction.  Input pieces, norm and SwiGLU epilogue as in gemv_b1.
  __device__ __forceinline__ bool gemv_b1_gu2(const mk_instr& in, int layer, const Gemv& g) {
    const int H = p.H, K = g.K, R = g.r1 - g.r0, nch = g.nch;
    const float* src = p.xres + (size_t)(2 * layer + 1) * H;
    const uint16_t* gain = p.layers[layer].mlp_norm;
    uint32_t own = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (warp + 8 * k < R) own |= 1u << k;
    if (!wait_counter(in.wait_idx, in.wait_count)) return false;
    if (tr) tr[1] = globaltimer();
    float4* xb = reinterpret_cast<float4*>(red);
    const uint32_t xs0 = smem_addr(red);
    const int pch = b1_piece_chunks(1);
    const bool narrow = K < kB1Chunk;
    float ag[8], au[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) ag[k] = au[k] = 0.f;
    for (int c0 = 0; c0 < nch; c0 += pch) {
      const int c1 = min(nch, c0 + pch);
      const uint32_t tag = ((uint32_t)layer << 12 | (uint32_t)OP_GATEUP << 6 | (uint32_t)(c0 / pch)) + 1u;
      if (ctl->xtag != tag) {
        if (c0 > 0) consumer_bar();  // every warp is done with the previous piece
        float ss = 0.f;
        for (int f = t; f < (c1 - c0) * 64; f += kConsumerThreads) {
          const int col = c0 * kB1Chunk + 4 * f;
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (col < K) {
            v = __ldcg(reinterpret_cast<const float4*>(src + col));
            const uint2 gv = __ldg(reinterpret_cast<const uint2*>(gain + col));
            ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
            v.x *= bf16_lo(gv.x);
            v.y *= bf16_hi(gv.x);
            v.z *= bf16_lo(gv.y);
            v.w *= bf16_hi(gv.y);
          }
          const int ff = f & 63;
          xb[((f >> 6) * 2 + (ff & 1)) * 32 + (ff >> 1)] = v;
        }
        ss = warp_sum(ss);
        if (lane == 0) ctl->sred[warp] = ss;
        consumer_bar();
        if (t == 0) {
          float s2 = 0.f;
#pragma unroll
          for (int w2 = 0; w2 < kConsumerWarps; ++w2) s2 += ctl->sred[w2];
          ctl->xss = (c0 == 0 ? 0.f : ctl->xss) + s2;  // pieces of the same input, in order
          ctl->xtag = tag;
        }
        consumer_bar();
      }
      if (tr && c0 == 0) tr[4] = globaltimer();
#pragma unroll 1
      for (int c = c0; c < c1; ++c) {
        const uint32_t xa = xs0 + (uint32_t)((c - c0) * 2 * 32 + lane) * 16u;
        const float4 x0 = lds_f4(xa), x1 = lds_f4(xa + 512u);
        const unsigned long long xp[4] = {pack2(x0.x, x0.y), pack2(x0.z, x0.w), pack2(x1.x, x1.y),
                                          pack2(x1.z, x1.w)};
        const uint32_t lanes_ok = !narrow || c * kB1Chunk + lane * 8 < K;
#pragma unroll
        for (int grp = 0; grp < 2; ++grp) {  // the gate stage, then the up stage
          const uint8_t* w = wait_full();
          if (tr && c == 0 && grp == 0) tr[5] = globaltimer();
          const uint32_t wj = smem_addr(w) + (uint32_t)(warp * kB1LineBytes + lane * 16);
          uint4 wv[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) wv[k] = lds_u4_if(wj + (uint32_t)(8 * k) * kB1LineBytes, ((own >> k) & 1u) & lanes_ok);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float d = sum2(dot8x2(wv[k], xp, 0ull));
            if (grp == 0)
              ag[k] += d;
            else
              au[k] += d;
          }
          release();
        }
      }
    }
    if (tr) tr[6] = globaltimer();
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[k] = ag[k];
      v[8 + k] = au[k];
    }
    const float tot = warp_reduce_multi<16>(v, lane);     // item lane / 2 of this warp
    const float up = __shfl_xor_sync(0xffffffffu, tot, 16);  // item q + 8: the up line of neuron q
    const int q = lane >> 1;
    if ((lane & 1) == 0 && q < 8 && ((own >> q) & 1u)) {
      const float scale = 1.f / sqrtf(ctl->xss / (float)K + p.eps);
      const float gs = tot * scale, us = up * scale;
      p.act[g.r0 + warp + 8 * q] = gs / (1.f + expf(-gs)) * us;
    }
    return true;
  }

  // ---- GEMV, batch 1: row-stationary tiles ------------------------------------
  // Stage s holds chunks [s * ncs, ...) of every line of the instruction, each
  // line kB1Chunk bf16 weights (512 bytes); a stage holds at most 64 line
  // chunks, so each warp has at most 8 of them.  With ncs chunks per stage,
  // warp w takes chunk w % ncs of every stage and the lines w / ncs, w / ncs +
  // 8 / ncs, ... (gate/up: those neurons, each a gate line and an up line);
  // lane l covers the columns [8l, 8l + 8) of its chunk.  Partial dot products
  // stay in registers (packed fp32 pairs) across all stages; at the end each
  // warp reduces its lines across its lanes, and the ncs warps that share a
  // line add their sums in a fixed order.  The input vector (fp32; times the
  // RMSNorm gain for the norm-fused ops) is in the reduction buffer, loaded
  // with one round trip to L2 per piece of kB1XPieceFloats columns and kept
  // for the op's next instruction on this SM; the stream itself has no block
  // barrier.  The norm's 1/rms is constant along K, so it scales the outputs;
  // its sum of squares is taken from the same loads.
  template <bool NORM, bool GATED>
  __device__ __forceinline__ bool gemv_b1(const mk_instr& in, int op, int layer) {
    const Gemv g = gemv_geo(p, in, op, layer);
    if (GATED && g.split) return gemv_b1_gu2(in, layer, g);
    const int H = p.H, K = g.K, lines = g.lines, R = g.r1 - g.r0, nch = g.nch, NCS = g.ncs;
    const float* src;
    const uint16_t* gain = nullptr;
    if (op == OP_QKV) {
      src = p.xres + (size_t)(2 * layer) * H;
      gain = p.layers[layer].attn_norm;
    } else if (op == OP_OPROJ) {
      src = p.attn;
    } else if (op == OP_GATEUP) {
      src = p.xres + (size_t)(2 * layer + 1) * H;
      gain = p.layers[layer].mlp_norm;
    } else if (op == OP_DOWN) {
      src = p.act;
    } else {  // LM head
      src = p.xres + (size_t)(2 * p.L) * H;
      gain = p.final_norm;
    }
    const int LSTEP = kConsumerWarps / NCS;  // warps per chunk: a warp's lines are LSTEP apart
    const int cw = warp % NCS, lw = warp / NCS;
    // this warp's item k: gate/up, neuron lw + LSTEP (k & 3) (gate line for k < 4,
    // up line for k >= 4); otherwise line lw + LSTEP k.  own: the items that exist.
    uint32_t own = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (GATED ? lw + LSTEP * (k & 3) < R : lw + LSTEP * k < lines) own |= 1u << k;
    auto line_of = [&](int k) {
      return GATED ? (k < 4 ? 0 : R) + lw + LSTEP * (k & 3) : lw + LSTEP * k;
    };
    // output rows: with one chunk per stage every warp finishes its own lines
    // (writer lanes: the reduced item lane / 4); otherwise thread t < rows
    // finishes row t from the per-warp sums
    const int q = lane >> 2;
    const bool writer = (lane & 3) == 0;
    int orow = -1;
    if (NCS == 1) {
      if (writer && (GATED ? q < 4 : true) && ((own >> q) & 1u)) orow = g.r0 + lw + LSTEP * (q & (GATED ? 3 : 7));
    } else if (t < R) {
      orow = g.r0 + t;
    }
    if (!wait_counter(in.wait_idx, in.wait_count)) return false;
    if (tr) tr[1] = globaltimer();
    // residual row of the epilogue, fetched before the stream
    float resid = 0.f;
    if ((op == OP_OPROJ || op == OP_DOWN) && orow >= 0)
      resid = __ldcg(p.xres + (size_t)(2 * layer + (op == OP_DOWN ? 1 : 0)) * H + orow);
    // input piece: [chunk][half][lane] float4 (lane l's 8 columns of a chunk in two halves)
    float4* xb = reinterpret_cast<float4*>(red);
    const uint32_t xs0 = smem_addr(red);
    const int pch = kB1XPieceFloats / kB1Chunk / NCS * NCS;  // chunks per piece, whole stages
    const bool narrow = K < kB1Chunk;  // lines are K wide: lanes past K hold stale bytes
    unsigned long long acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0ull;  // (+0.0f, +0.0f) pairs
    int s = 0;  // stage
    for (int c0 = 0; c0 < nch; c0 += pch) {
      const int c1 = min(nch, c0 + pch);
      const uint32_t tag = ((uint32_t)layer << 12 | (uint32_t)op << 6 | (uint32_t)(c0 / pch)) + 1u;
      if (ctl->xtag != tag) {
        if (c0 > 0) consumer_bar();  // every warp is done with the previous piece
        float ss = 0.f;
        for (int f = t; f < (c1 - c0) * 64; f += kConsumerThreads) {
          const int col = c0 * kB1Chunk + 4 * f;
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (col < K) {
            v = __ldcg(reinterpret_cast<const float4*>(src + col));
            if (NORM) {
              const uint2 gv = __ldg(reinterpret_cast<const uint2*>(gain + col));
              ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
              v.x *= bf16_lo(gv.x);
              v.y *= bf16_hi(gv.x);
              v.z *= bf16_lo(gv.y);
              v.w *= bf16_hi(gv.y);
            }
          }
          const int ff = f & 63;
          xb[((f >> 6) * 2 + (ff & 1)) * 32 + (ff >> 1)] = v;
        }
        if (NORM) {
          ss = warp_sum(ss);
          if (lane == 0) ctl->sred[warp] = ss;
        }
        consumer_bar();
        if (t == 0) {
          if (NORM) {
            float s2 = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < kConsumerWarps; ++w2) s2 += ctl->sred[w2];
            ctl->xss = (c0 == 0 ? 0.f : ctl->xss) + s2;  // pieces of the same input, in order
          }
          ctl->xtag = tag;
        }
        consumer_bar();
      }
      if (tr && c0 == 0) tr[4] = globaltimer();
      const int s1 = (c1 + NCS - 1) / NCS;
#pragma unroll 1
      for (; s < s1; ++s) {
        const uint8_t* w = wait_full();
        if (tr && s == 0) tr[5] = globaltimer();
        const int c = s * NCS + cw;  // this warp's chunk
        if (c < nch) {
          // every load of the stage first (x, then the warp's own lines), then the arithmetic;
          // shared-space loads on 32-bit shared addresses
          const uint32_t xa = xs0 + (uint32_t)((c - c0) * 2 * 32 + lane) * 16u;
          const float4 x0 = lds_f4(xa), x1 = lds_f4(xa + 512u);
          const uint32_t wj = smem_addr(w) + (uint32_t)(cw * lines * kB1LineBytes + lane * 16);
          // items the warp does not own (and, for a K narrower than a chunk, the
          // lanes past K) load zeros: no branch, so the eight chains interleave
          const uint32_t lanes_ok = !narrow || c * kB1Chunk + lane * 8 < K;
          uint4 wv[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            wv[k] = lds_u4_if(wj + (uint32_t)line_of(k) * kB1LineBytes, ((own >> k) & 1u) & lanes_ok);
          const unsigned long long xp[4] = {pack2(x0.x, x0.y), pack2(x0.z, x0.w), pack2(x1.x, x1.y),
                                            pack2(x1.z, x1.w)};
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] = dot8x2(wv[k], xp, acc[k]);
        }
        release();
      }
    }
    if (tr) tr[6] = globaltimer();
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = sum2(acc[k]);
    float tot = warp_reduce_multi<8>(v, lane);  // item lane / 4 of this warp
    float up = GATED ? __shfl_xor_sync(0xffffffffu, tot, 16) : 0.f;  // item q + 4: the up line of neuron q
    if (NCS > 1) {
      // the warps sharing a line add their sums in chunk order
      if (writer && ((own >> q) & 1u) && (GATED ? q < 4 : true)) {
        const int li = lw + LSTEP * (q & (GATED ? 3 : 7));
        ctl->b1red[li * 4 + cw] = tot;
        if (GATED) ctl->b1red[(kB1MaxLines / 2 + li) * 4 + cw] = up;
      }
      consumer_bar();
      tot = up = 0.f;
      if (orow >= 0) {
        const int li = t;
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
          if (c2 >= NCS) break;
          tot += ctl->b1red[li * 4 + c2];
          if (GATED) up += ctl->b1red[(kB1MaxLines / 2 + li) * 4 + c2];
        }
      }
    }
    const float scale = NORM ? 1.f / sqrtf(ctl->xss / (float)K + p.eps) : 1.f;
    const bool amx = op == OP_LMHEAD && p.argmax;
    unsigned long long best = 0ull;
    if (orow >= 0) {
      if (GATED) {
        const float gs = tot * scale, us = up * scale;
        p.act[orow] = gs / (1.f + expf(-gs)) * us;
      } else {
        const float y = tot * scale;
        if (op == OP_QKV) {
          p.qkv[orow] = y;  // q | k | v concatenated, like the instruction's rows
        } else if (op == OP_OPROJ) {
          p.xres[(size_t)(2 * layer + 1) * H + orow] = resid + y;
        } else if (op == OP_DOWN) {
          p.xres[(size_t)(2 * layer + 2) * H + orow] = resid + y;
        } else {
          p.logits[orow] = y;
          if (amx) best = argmax_key(y, orow);
        }
      }
    }
    if (amx) {  // the instruction's arg-max: warps, then shared memory, then one global atomic
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, off));
      if (lane == 0) atomicMax(&ctl->amax[0], best);
      consumer_bar();
      if (t == 0) {
        atomicMax(p.argmax, ctl->amax[0]);
        ctl->amax[0] = 0ull;
      }
    }
    return true;
  }

  // ---- GEMV, batch > 1: tensor cores ---------------------------------------
  // mma.m16n8k16 with A = a stage tile of 16 weight rows (ldmatrix from the
  // ring), B = the bf16 inputs of the batch (n = sequence, columns b >= B are
  // zero), D[row][b] in fp32 registers.  Warps split each chunk's k-steps
  // between them and keep every tile's partial sums in registers for the
  // whole instruction; one cross-warp reduction in a fixed order ends it.
  // The inputs of a chunk are fragments in registers, loaded (fp32, from L2)
  // one chunk ahead.  RMSNorm: the gain is applied to the inputs, and the
  // per-sequence 1/rms factor, whose sum of squares accumulates from the same
  // loads, scales the outputs in the epilogue (it is constant along K).
  //
  // MoE: the router and the expert gate/up read the MLP input like gate/up;
  // expert down runs K over the picked experts (slot after slot), its inputs
  // being each slot's SwiGLU output times the sequence's routing weight.
  // `slot` is the expert slot of a gate/up piece; wait_idx < 0: no wait.
  template <bool NORM, bool GATED>
  __device__ __forceinline__ bool gemv_tc(const Gemv& g, int op, int layer, int wait_idx, int wait_count, int slot) {
    constexpr int TR = GATED ? 8 : 16;  // output rows per tile
    constexpr int MAXT = (GATED ? kBatchedMaxRowsGated : (NORM ? kBatchedMaxRows : kBatchedMaxRowsLongK)) / TR;
    constexpr int KPW = kBChunk / 16 / kConsumerWarps;  // k-steps per warp per chunk
    const int B = p.B, BH = B * p.H, nrows = g.r1 - g.r0, ntiles = g.bnt;
    const bool moe_down = op == OP_EXP_DOWN;
    const int nd = moe_down ? moe_down_chunks(p) : 1;
    const float* src;
    const uint16_t* gain = nullptr;
    int ld;  // elements per sequence in src
    if (op == OP_QKV) {
      src = p.xres + (size_t)(2 * layer) * BH, gain = p.layers[layer].attn_norm, ld = p.H;
    } else if (op == OP_GATEUP || op == OP_ROUTER || op == OP_EXP_GATEUP) {
      src = p.xres + (size_t)(2 * layer + 1) * BH, gain = p.layers[layer].mlp_norm, ld = p.H;
    } else if (!NORM) {
      src = nullptr, ld = 0;  // o_proj, down, expert down: bf16 inputs, staged below
    } else {
      src = p.xres + (size_t)(2 * p.L) * BH, gain = p.final_norm, ld = p.H;
    }
    if (wait_idx >= 0) {
      if (!wait_counter(wait_idx, wait_count)) return false;
      if (tr) tr[1] = globaltimer();
    }
    const int gq = lane >> 2, cq = lane & 3;
    const bool bval = gq < B;  // this lane's B-fragment column (sequence gq) exists
    const float* xrow = NORM ? src + (size_t)(bval ? gq : 0) * ld : nullptr;
    // columns of chunk j
    auto cols = [&](int j) { return moe_down ? min(kBChunk, p.Ie - (j % nd) * kBChunk) : min(kBChunk, g.K - j * kBChunk); };
    float acc[MAXT][4];
#pragma unroll
    for (int t2 = 0; t2 < MAXT; ++t2) acc[t2][0] = acc[t2][1] = acc[t2][2] = acc[t2][3] = 0.f;
    // ldmatrix row address of this lane within a stage: A-row R = lane & 15
    // lives in box R >> 3 as row r = R & 7; k-step ks = warp + 8 kk reads
    // column block (warp >> 2) + 2 kk, 16-byte chunk ((warp & 3) << 1) | (lane >> 4),
    // stored at chunk position (chunk ^ r) of its 128-byte line.
    const uint32_t rr7 = (uint32_t)(lane & 7), ch = ((uint32_t)(warp & 3) << 1) | (uint32_t)(lane >> 4);
    const uint32_t lrow = (uint32_t)((lane >> 3) & 1) * kBBoxBytes + (uint32_t)(warp >> 2) * 1024u + rr7 * 128u +
                          ((ch ^ rr7) << 4);
    float ss = 0.f;
    if constexpr (NORM) {
      // K = hidden: few chunks of many tiles.  fp32 inputs (and gains) of the
      // next chunk load into registers while this one streams.
      float2 xr[KPW][2];
      uint32_t gr[KPW][2];
      uint32_t xf[KPW][2];
      auto load = [&](int j) {
        const int nks = cols(j) / 16;
#pragma unroll
        for (int kk = 0; kk < KPW; ++kk) {
          const int ks = warp + kk * kConsumerWarps;
          const int k = j * kBChunk + ks * 16 + 2 * cq;
          if (bval && ks < nks) {
            xr[kk][0] = __ldcg(reinterpret_cast<const float2*>(xrow + k));
            xr[kk][1] = __ldcg(reinterpret_cast<const float2*>(xrow + k + 8));
            gr[kk][0] = __ldg(reinterpret_cast<const unsigned int*>(gain + k));
            gr[kk][1] = __ldg(reinterpret_cast<const unsigned int*>(gain + k + 8));
          } else {
            xr[kk][0] = xr[kk][1] = make_float2(0.f, 0.f);
            gr[kk][0] = gr[kk][1] = 0u;
          }
        }
      };
      load(0);
      for (int j = 0; j < g.bnch; ++j) {
        const int nks = cols(j) / 16;
#pragma unroll
        for (int kk = 0; kk < KPW; ++kk) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float2 x = xr[kk][h];
            ss = fmaf(x.x, x.x, fmaf(x.y, x.y, ss));
            xf[kk][h] = pack_bf16x2(x.x * bf16_lo(gr[kk][h]), x.y * bf16_hi(gr[kk][h]));
          }
        }
        if (tr && j == 0) tr[4] = globaltimer();
        if (j + 1 < g.bnch) load(j + 1);
#pragma unroll
        for (int t2 = 0; t2 < MAXT; ++t2) {
          if (t2 < ntiles) {
            const uint32_t st = smem_addr(wait_full()) + lrow;
            if (tr && j == 0 && t2 == 0) tr[5] = globaltimer();
#pragma unroll
            for (int kk = 0; kk < KPW; ++kk) {
              const int ks = warp + kk * kConsumerWarps;
              if (ks < nks) {
                uint32_t a[4];
                ldmatrix_x4(a, st + (uint32_t)kk * 2048u);
                mma16816(acc[t2], a[0], a[1], a[2], a[3], xf[kk][0], xf[kk][1]);
              }
            }
            release();
          }
        }
      }
    } else {
      // Long K over few rows (o_proj, down, expert down): a chunk may be one
      // tile, shorter than an L2 round trip.  The chunks' bf16 inputs stream
      // into a shared-memory ring with cp.async, two chunks ahead; the ring
      // is [slot][sequence][column] at a padded pitch (conflict-free
      // fragment reads), in the reduction buffer.
      const uint16_t* xsrc = op == OP_OPROJ ? p.attn_bf : (moe_down ? p.moe_act : p.act_bf);
      const int xld = op == OP_OPROJ ? p.nq * p.hd : (moe_down ? p.Ie : p.I);
      uint8_t* xs = reinterpret_cast<uint8_t*>(red);
      auto stage_x = [&](int j) {  // chunk j into ring slot j % kXsSlots (this thread's pieces)
        const int c16 = cols(j) / 8;  // 16-byte pieces per sequence
        const uint16_t* s0 = moe_down ? xsrc + (size_t)(j / nd) * B * p.Ie + (j % nd) * kBChunk
                                      : xsrc + (size_t)j * kBChunk;
        uint8_t* d0 = xs + (size_t)(j % kXsSlots) * kMaxBatch * kXsPitchBytes;
        for (int idx = t; idx < B * c16; idx += kConsumerThreads) {
          const int b = idx / c16, c = idx % c16;
          cp_async16(d0 + (size_t)b * kXsPitchBytes + c * 16, s0 + (size_t)b * xld + c * 8);
        }
      };
      stage_x(0);
      cp_async_commit();
      if (g.bnch > 1) stage_x(1);
      cp_async_commit();
      if (tr) tr[4] = globaltimer();
      const uint32_t xrd = (uint32_t)gq * kXsPitchBytes + (uint32_t)cq * 4u;  // this lane's fragment row
      for (int j = 0; j < g.bnch; ++j) {
        const int nks = cols(j) / 16;
        cp_async_wait<1>();  // chunk j landed (only chunk j + 1 may be pending)
        consumer_bar();      // ... for every thread's pieces; every warp is done with chunk j - 1
        if (j + 2 < g.bnch) stage_x(j + 2);  // into chunk j - 1's slot
        cp_async_commit();
        const uint32_t xb = smem_addr(xs + (size_t)(j % kXsSlots) * kMaxBatch * kXsPitchBytes) + xrd;
#pragma unroll
        for (int t2 = 0; t2 < MAXT; ++t2) {
          if (t2 < ntiles) {
            const uint32_t st = smem_addr(wait_full()) + lrow;
            if (tr && j == 0 && t2 == 0) tr[5] = globaltimer();
#pragma unroll
            for (int kk = 0; kk < KPW; ++kk) {
              const int ks = warp + kk * kConsumerWarps;
              if (ks < nks) {
                uint32_t a[4], b0, b1;
                ldmatrix_x4(a, st + (uint32_t)kk * 2048u);
                asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b0) : "r"(xb + (uint32_t)ks * 32u));
                asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b1) : "r"(xb + (uint32_t)ks * 32u + 16u));
                mma16816(acc[t2], a[0], a[1], a[2], a[3], b0, b1);
              }
            }
            release();
          }
        }
      }
      consumer_bar();  // the ring (the reduction buffer) is free for the reduction below
    }
    if (tr) tr[6] = globaltimer();
    if (NORM) {
      // per-warp sum of squares of sequence gq (lanes cq = 0..3 hold disjoint columns)
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      if (cq == 0) ctl->aml[warp * kMaxBatch + gq] = ss;
    }
    // Cross-warp reduction, four tiles per round: warp w's partials of a tile
    // at red[w * 512 + q * 128 + lane * 4 + e]; thread (q, l, i) then sums
    // accumulator elements i and i + 2 of lane l over the warps.
    const int q = t >> 6, l = (t >> 1) & 31, i = t & 1;
    const int lgq = l >> 2, b = 2 * (l & 3) + i;
    const bool amx = op == OP_LMHEAD && p.argmax;
    float sc = 1.f;
    const int qkvw = p.nq * p.hd + 2 * p.nkv * p.hd;
#pragma unroll
    for (int t0 = 0; t0 < MAXT; t0 += 4) {
      if (t0 < ntiles) {
        if (t0 > 0) consumer_bar();  // the previous round's sums are read
#pragma unroll
        for (int dq = 0; dq < 4; ++dq)
          if (t0 + dq < MAXT && t0 + dq < ntiles)
            *reinterpret_cast<float4*>(red + warp * 512 + dq * 128 + lane * 4) =
                make_float4(acc[t0 + dq][0], acc[t0 + dq][1], acc[t0 + dq][2], acc[t0 + dq][3]);
        consumer_bar();
        if (NORM && t0 == 0 && b < B) {
          float tot = 0.f;
          for (int w = 0; w < kConsumerWarps; ++w) tot += ctl->aml[w * kMaxBatch + b];
          sc = 1.f / sqrtf(tot / (float)g.K + p.eps);
        }
        const int tile = t0 + q;
        if (tile < ntiles && b < B) {
          float v0 = 0.f, v1 = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            v0 += red[w * 512 + q * 128 + l * 4 + i];
            v1 += red[w * 512 + q * 128 + l * 4 + 2 + i];
          }
          v0 *= sc;
          v1 *= sc;
          if (GATED) {
            const int row = tile * TR + lgq;  // v0 = gate, v1 = up of neuron row
            if (row < nrows) {
              const float a = v0 / (1.f + expf(-v0)) * v1;
              if (op == OP_EXP_GATEUP)  // weighted by the sequence's routing weight of the slot
                p.moe_act[((size_t)slot * B + b) * p.Ie + (g.r0 - ctl->moe_uniq[slot] * p.Ie) + row] =
                    f32_to_bf16_bits(a * ctl->moe_tw[slot][b]);
              else
                p.act_bf[(size_t)b * p.I + g.r0 + row] = f32_to_bf16_bits(a);
            }
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int rr = tile * TR + lgq + 8 * h;
              if (rr < nrows) {
                const float y = h ? v1 : v0;
                const int row = g.r0 + rr;
                if (op == OP_QKV) {
                  p.qkv[(size_t)b * qkvw + row] = y;
                } else if (op == OP_OPROJ) {
                  const size_t o = (size_t)b * p.H + row;
                  p.xres[(size_t)(2 * layer + 1) * BH + o] = __ldcg(p.xres + (size_t)(2 * layer) * BH + o) + y;
                } else if (op == OP_DOWN || moe_down) {
                  const size_t o = (size_t)b * p.H + row;
                  p.xres[(size_t)(2 * layer + 2) * BH + o] = __ldcg(p.xres + (size_t)(2 * layer + 1) * BH + o) + y;
                } else if (op == OP_ROUTER) {
                  p.moe_router[((size_t)layer * B + b) * p.E + row] = y;
                } else {
                  p.logits[(size_t)b * p.V + row] = y;
                  if (amx) atomicMax(&ctl->amax[b], argmax_key(y, row));
                }
              }
            }
          }
        }
      }
    }
    if (amx) {  // the instruction's arg-max per sequence (shared atomics above), one global atomic each
      consumer_bar();
      if (t < B) {
        atomicMax(p.argmax + t, ctl->amax[t]);
        ctl->amax[t] = 0ull;
      }
    }
    return true;
  }

  __device__ __forceinline__ bool gemv(const mk_instr& in, int op, int layer) {
    if constexpr (BATCHED) {
      Gemv g = gemv_geo(p, in, op, layer);
      if (op == OP_EXP_DOWN) g.bnch = ctl->moe_count * moe_down_chunks(p);  // routing of this layer, in place
      if (op == OP_GATEUP) return gemv_tc<true, true>(g, op, layer, in.wait_idx, in.wait_count, -1);
      if (op == OP_QKV || op == OP_LMHEAD || op == OP_ROUTER)
        return gemv_tc<true, false>(g, op, layer, in.wait_idx, in.wait_count, -1);
      return gemv_tc<false, false>(g, op, layer, in.wait_idx, in.wait_count, -1);
    }
    if (op == OP_GATEUP) return gemv_b1<true, true>(in, op, layer);
    if (op == OP_QKV || op == OP_LMHEAD) return gemv_b1<true, false>(in, op, layer);
    return gemv_b1<false, false>(in, op, layer);
  }

  // ---- MoE routing ---------------------------------------------------------------
  // Top-k of each sequence's router logits (the larger logit first, a tie to
  // the lower expert index; Shazeer et al. 2017, sparsely-gated mixture of
  // experts), weights = softmax over the k picked logits, and the distinct
  // picked experts in ascending order as slots.  Every SM computes the same
  // routing from the same logits; the SM of slot instruction 0 writes it out.
  __device__ __forceinline__ void moe_select(int layer, bool dump) {
    const int E = p.E, K = p.topk, B = p.B;
    if (t < kMaxExperts / 32) ctl->moe_mask[t] = 0u;
    for (int i = t; i < kMaxSel * kMaxBatch; i += kConsumerThreads) (&ctl->moe_tw[0][0])[i] = 0.f;
    consumer_bar();
    int pick = 0;    // lane j < K of warp b < B: the j-th pick of sequence b
    float pw = 0.f;  // and its weight
    if (warp < B) {
      const float* r = p.moe_router + ((size_t)layer * B + warp) * E;
      float v[kMaxExperts / 32];
#pragma unroll
      for (int q = 0; q < kMaxExperts / 32; ++q) {
        const int e = lane + 32 * q;
        const float x = e < E ? __ldcg(r + e) : -INFINITY;
        v[q] = x != x ? -INFINITY : x;  // NaN ranks below every number
      }
      uint32_t taken = 0u;
      float top0 = 0.f, den = 0.f, mine = 0.f;
      for (int j = 0; j < K; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < kMaxExperts / 32; ++q) {
          const int e = lane + 32 * q;
          if (e < E && !((taken >> q) & 1u) && (v[q] > bv || (v[q] == bv && e < bi))) {
            bv = v[q];
            bi = e;
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
          }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (j == 0) top0 = bv;
        const float ex = expf(bv - top0);
        den += ex;
        if (lane == j) {
          pick = bi;
          mine = ex;
        }
      }
      if (lane < K) {
        pw = mine / den;
        atomicOr(&ctl->moe_mask[pick >> 5], 1u << (pick & 31));
        if (dump) {
          p.moe_sel[((size_t)layer * B + warp) * K + lane] = pick;
          p.moe_selw[((size_t)layer * B + warp) * K + lane] = pw;
        }
      }
    }
    consumer_bar();
    // slot of a picked expert: the picked experts below it
    auto slot_of = [&](int e) {
      int sl = 0;
      for (int w = 0; w < (e >> 5); ++w) sl += __popc(ctl->moe_mask[w]);
      return sl + __popc(ctl->moe_mask[e >> 5] & ((1u << (e & 31)) - 1u));
    };
    if (t < E && ((ctl->moe_mask[t >> 5] >> (t & 31)) & 1u)) ctl->moe_uniq[slot_of(t)] = (int16_t)t;
    if (t == 0) {
      int c = 0;
      for (int w = 0; w < kMaxExperts / 32; ++w) c += __popc(ctl->moe_mask[w]);
      ctl->moe_count = c;
      if (dump) p.moe_count[layer] = c;
    }
    if (warp < B && lane < K) ctl->moe_tw[slot_of(pick)][warp] = pw;
    consumer_bar();
    if (t == 0) {  // hand the routing to the producer
      __threadfence_block();
      *(volatile int*)&ctl->moe_pub = layer + 1;
    }
  }

  // One expert gate/up slot: wait for the router, route, then this slot's
  // even share of the (picked expert, 8-neuron tile) units, piece by piece.
  __device__ __forceinline__ bool moe_gateup(const mk_instr& in, int layer) {
    if constexpr (BATCHED) {
      if (!wait_counter(in.wait_idx, in.wait_count)) return false;
      if (tr) tr[1] = globaltimer();
      moe_select(layer, in.a == 0);
      const int64_t U = (int64_t)ctl->moe_count * (p.Ie / 8);
      const int64_t g1 = even_begin(U, in.b, in.a + 1);
      for (int64_t g = even_begin(U, in.b, in.a); g < g1;) {
        int sl;
        const Gemv gm = moe_gate_piece(p, ctl, layer, g, g1, &sl);
        if (!gemv_tc<true, true>(gm, OP_EXP_GATEUP, layer, -1, 0, sl)) return false;
        g += gm.bnt;
        consumer_bar();  // the reduction buffer is free for the next piece
      }
      return true;
    } else {
      return false;  // MoE runs on the tensor-core kernel only
    }
  }

  // ---- attention ---------------------------------------------------------------
  // Batch 1: the cached positions of one piece on the CUDA cores, in fp32.  A
  // stage holds P positions of K (or V) as [64-column block][position][64]
  // with the 128-byte swizzle (16-byte chunk c of position row r at chunk
  // position c ^ (r & 7)).  Warp w takes positions [w P/8, (w + 1) P/8) of
  // every stage with its own online softmax (log2 units; q pre-scaled by
  // log2(e)/sqrt(hd)).  Lane l covers the 8 dimensions (l % DS) * 8 .. + 8
  // (DS = HD / 8) of the positions of its group l / DS: scores take the dot
  // products of those slices, reduced over the DS lanes by halving shuffles;
  // P.V accumulates o[head][its 8 dims] over its group's positions in packed
  // fp32 pairs.  At the end the position groups of a warp, then the warps,
  // merge into the piece's partial, the same partial the tensor-core path
  // writes.
  template <int HD, int G>
  __device__ __forceinline__ void attn_ff(const Attn& a, int q0) {
    constexpr int P = kStageBytes / (HD * 2);  // positions per stage
    constexpr int DS = HD / 8;                 // lanes per position (8 dimensions each)
    constexpr int PG = 32 / DS;                // position groups per warp
    constexpr int PW = P / kConsumerWarps;     // positions per warp per stage
    constexpr int NPL = PW / PG;               // positions per lane per stage (8)
    constexpr int NB = 4;                      // positions per score batch
    constexpr int VB = G * NB;                 // score values per batch (<= 16)
    constexpr int RR = VB < DS ? VB : DS;      // values per reduction round
    constexpr uint32_t CBB = (uint32_t)P * 128u;
    constexpr int NJ = (G * PW + 31) / 32;     // softmax entries per lane
    static_assert(NPL % NB == 0 && VB % RR == 0, "attention tiling");
    const int ds = lane % DS, pg = lane / DS;
    const uint32_t blk = (uint32_t)(ds >> 3) * CBB, chunk = (uint32_t)(ds & 7);
    // q slices of the G heads (fp32 pairs)
    unsigned long long qp[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float4 q0v = *reinterpret_cast<const float4*>(ctl->qs + h * HD + ds * 8);
      const float4 q1v = *reinterpret_cast<const float4*>(ctl->qs + h * HD + ds * 8 + 4);
      qp[h][0] = pack2(q0v.x, q0v.y);
      qp[h][1] = pack2(q0v.z, q0v.w);
      qp[h][2] = pack2(q1v.x, q1v.y);
      qp[h][3] = pack2(q1v.z, q1v.w);
    }
    unsigned long long o[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0ull;
    float m[G], l[G];
#pragma unroll
    for (int h = 0; h < G; ++h) m[h] = -1e30f, l[h] = 0.f;
    // this warp's scores / probabilities of a stage, [position][4 heads]
    float* S = red + kRedFloats + warp * (PW * 4);
    for (int s = 0; s < a.nsub; ++s) {
      const int np = min(P, a.n_cached - s * P);
      const uint32_t Ks = smem_addr(wait_stage(k));
      const uint32_t Vs = smem_addr(wait_stage(k + 1));
      if (tr && s == 0) tr[5] = globaltimer();
      // -- scores of the lane's positions, NB at a time, reduced over the DS lanes
#pragma unroll
      for (int i0 = 0; i0 < NPL; i0 += NB) {
        float part[VB];
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          const int pos = warp * PW + pg + PG * (i0 + i);
          const uint4 kv = lds_u4_if(Ks + blk + (uint32_t)pos * 128u + ((chunk ^ (uint32_t)(pos & 7)) << 4), pos < np);
          const unsigned long long kp[4] = {pack2(bf16_lo(kv.x), bf16_hi(kv.x)), pack2(bf16_lo(kv.y), bf16_hi(kv.y)),
                                            pack2(bf16_lo(kv.z), bf16_hi(kv.z)), pack2(bf16_lo(kv.w), bf16_hi(kv.w))};
#pragma unroll
          for (int h = 0; h < G; ++h) {
            unsigned long long d = ffma2(kp[0], qp[h][0], 0ull);
            d = ffma2(kp[1], qp[h][1], d);
            d = ffma2(kp[2], qp[h][2], d);
            d = ffma2(kp[3], qp[h][3], d);
            part[h * NB + i] = sum2(d);
          }
        }
#pragma unroll
        for (int r = 0; r < VB / RR; ++r) {
          float v[RR];
#pragma unroll
          for (int e = 0; e < RR; ++e) v[e] = part[r * RR + e];
          const float tot = group_reduce_multi<RR, DS>(v, lane);  // value index (ds) >> log2(DS / RR)
          const int vi = r * RR + (ds >> (ilog2c(DS) - ilog2c(RR)));
          if ((ds & (DS / RR - 1)) == 0) {
            const int h = vi / NB, i = vi % NB;
            const int pl = pg + PG * (i0 + i);  // the position within the warp's share
            S[pl * 4 + h] = warp * PW + pl < np ? tot : -1e30f;
          }
        }
      }
      __syncwarp();
      // -- online softmax per head over the warp's PW positions: lane j handles
      // entries j, j + 32, ... of [head][position]
      float mt[G];
#pragma unroll
      for (int h = 0; h < G; ++h) mt[h] = -1e30f;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int idx = lane + 32 * j, h = min(idx / PW, G - 1), pl = idx % PW;
        float x = idx < G * PW ? S[pl * 4 + h] : -1e30f;
#pragma unroll
        for (int off = PW / 2; off; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
          if (hh == h) mt[hh] = x;
      }
      // each head's maximum lives in the lanes of its entries: broadcast
      float c[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mx = __shfl_sync(0xffffffffu, mt[h], (h * PW) % 32);
        const float mn = fmaxf(m[h], mx);
        c[h] = exp2f(m[h] - mn);
        m[h] = mn;
      }
      float lt[G];
#pragma unroll
      for (int h = 0; h < G; ++h) lt[h] = 0.f;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int idx = lane + 32 * j, h = min(idx / PW, G - 1), pl = idx % PW;
        float mh = m[0];
#pragma unroll
        for (int hh = 1; hh < G; ++hh)
          if (hh == h) mh = m[hh];
        const bool act = idx < G * PW;
        const float sc = act ? S[pl * 4 + h] : -1e30f;
        const float pv = act && warp * PW + pl < np ? exp2f(sc - mh) : 0.f;
        if (act) S[pl * 4 + h] = pv;
        float y = pv;
#pragma unroll
        for (int off = PW / 2; off; off >>= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
          if (hh == h) lt[hh] = y;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) l[h] = l[h] * c[h] + __shfl_sync(0xffffffffu, lt[h], (h * PW) % 32);
      __syncwarp();
      // -- o = o * c + P . V over the lane's positions
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const unsigned long long cc = pack2(c[h], c[h]);
#pragma unroll
        for (int e = 0; e < 4; ++e) o[h][e] = ffma2(o[h][e], cc, 0ull);
      }
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int pl = pg + PG * i, pos = warp * PW + pl;
        const uint4 vv = lds_u4_if(Vs + blk + (uint32_t)pos * 128u + ((chunk ^ (uint32_t)(pos & 7)) << 4), pos < np);
        const float4 pr = *reinterpret_cast<const float4*>(S + pl * 4);
        const unsigned long long vp[4] = {pack2(bf16_lo(vv.x), bf16_hi(vv.x)), pack2(bf16_lo(vv.y), bf16_hi(vv.y)),
                                          pack2(bf16_lo(vv.z), bf16_hi(vv.z)), pack2(bf16_lo(vv.w), bf16_hi(vv.w))};
        const float ph[4] = {pr.x, pr.y, pr.z, pr.w};
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const unsigned long long pp = pack2(ph[h], ph[h]);
#pragma unroll
          for (int e = 0; e < 4; ++e) o[h][e] = ffma2(vp[e], pp, o[h][e]);
        }
      }
      __syncwarp();
      release();  // K slot
      release();  // V slot
    }
    if (tr) tr[6] = globaltimer();
    // -- the position groups of each warp: one o per warp (m, l are warp-uniform)
#pragma unroll
    for (int off = DS; off < 32; off <<= 1)
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x, y;
          asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(o[h][e]));
          x += __shfl_xor_sync(0xffffffffu, x, off);
          y += __shfl_xor_sync(0xffffffffu, y, off);
          o[h][e] = pack2(x, y);
        }
    if (a.owns_new && warp == 0) {
      // the new token: its score for every head (the DS lanes of group 0 hold
      // its dimension slices), folded into warp 0's state
      const uint4 kv = *reinterpret_cast<const uint4*>(ctl->knew + ds * 8);
      const unsigned long long kp[4] = {pack2(bf16_lo(kv.x), bf16_hi(kv.x)), pack2(bf16_lo(kv.y), bf16_hi(kv.y)),
                                        pack2(bf16_lo(kv.z), bf16_hi(kv.z)), pack2(bf16_lo(kv.w), bf16_hi(kv.w))};
      const uint4 vv = *reinterpret_cast<const uint4*>(ctl->vnew + ds * 8);
      const unsigned long long vp[4] = {pack2(bf16_lo(vv.x), bf16_hi(vv.x)), pack2(bf16_lo(vv.y), bf16_hi(vv.y)),
                                        pack2(bf16_lo(vv.z), bf16_hi(vv.z)), pack2(bf16_lo(vv.w), bf16_hi(vv.w))};
#pragma unroll
      for (int h = 0; h < G; ++h) {
        unsigned long long d = ffma2(kp[0], qp[h][0], 0ull);
        d = ffma2(kp[1], qp[h][1], d);
        d = ffma2(kp[2], qp[h][2], d);
        d = ffma2(kp[3], qp[h][3], d);
        float sn = sum2(d);
#pragma unroll
        for (int off = DS / 2; off; off >>= 1) sn += __shfl_xor_sync(0xffffffffu, sn, off);
        const float mn = fmaxf(m[h], sn);
        const float cc = exp2f(m[h] - mn), en = exp2f(sn - mn);
        m[h] = mn;
        l[h] = l[h] * cc + en;
        const unsigned long long c2 = pack2(cc, cc), e2 = pack2(en, en);
#pragma unroll
        for (int e = 0; e < 4; ++e) o[h][e] = ffma2(vp[e], e2, ffma2(o[h][e], c2, 0ull));
      }
    }
    // -- merge the warps through shared memory (one round: G heads fit)
    constexpr int HR = kRedFloats / (kConsumerWarps * HD) < G ? kRedFloats / (kConsumerWarps * HD) : G;
    static_assert(HR == G, "one merge round");
    const size_t pbase = ((size_t)a.b * p.nq + q0) * p.n_chunks + a.c;
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        ctl->aml[(warp * kMaxGroup + h) * 2] = m[h];
        ctl->aml[(warp * kMaxGroup + h) * 2 + 1] = l[h];
      }
    }
    if (pg == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float4 a0, a1;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(a0.x), "=f"(a0.y) : "l"(o[h][0]));
        asm("mov.b64 {%0, %1}, %2;" : "=f"(a0.z), "=f"(a0.w) : "l"(o[h][1]));
        asm("mov.b64 {%0, %1}, %2;" : "=f"(a1.x), "=f"(a1.y) : "l"(o[h][2]));
        asm("mov.b64 {%0, %1}, %2;" : "=f"(a1.z), "=f"(a1.w) : "l"(o[h][3]));
        *reinterpret_cast<float4*>(red + (warp * HR + h) * HD + ds * 8) = a0;
        *reinterpret_cast<float4*>(red + (warp * HR + h) * HD + ds * 8 + 4) = a1;
      }
    }
    consumer_bar();
    for (int id = t; id < G * HD; id += kConsumerThreads) {
      const int h = id / HD, d = id % HD;
      float M = -1e30f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, ctl->aml[(w * kMaxGroup + h) * 2]);
      float den = 0.f, num = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float cw = exp2f(ctl->aml[(w * kMaxGroup + h) * 2] - M);
        den = fmaf(cw, ctl->aml[(w * kMaxGroup + h) * 2 + 1], den);
        num = fmaf(cw, red[(w * HR + h) * HD + d], num);
      }
      if (a.npieces == 1) {  // the whole row: the output itself
        p.attn[(size_t)a.b * p.nq * HD + (size_t)(q0 + h) * HD + d] = num / den;
      } else {
        const size_t pi = pbase + (size_t)h * p.n_chunks;
        p.part_o[pi * HD + d] = num;
        if (d == 0) {
          p.part_ml[pi * 2] = M;
          p.part_ml[pi * 2 + 1] = den;
        }
      }
    }
    consumer_bar();
  }

  // Batch > 1: the cached positions of one chunk on tensor cores.  A stage is
  // a TMA box of P positions, [64-column block][position][64] with the 128-byte
  // swizzle.  Warp w owns key tiles of 16 positions of every stage:
  //   S^T[key][head] = K[key][:] . q[head][:]   mma: A = K tile (ldmatrix),
  //                                              B = q (bf16, heads >= G zero)
  //   O^T[dim][head] += V[key][dim]^T P^T        mma: A = V tile (ldmatrix.trans),
  //                                              B = P (movmatrix transposes S's layout)
  // with its own online softmax (log2 units, q pre-scaled by log2(e)/sqrt(hd)).
  // The warps' (m, l, o) are merged through shared memory into the chunk's
  // partial, the same partial the CUDA-core path writes.
  template <int HD, int G>
  __device__ __forceinline__ void attn_tc(const Attn& a, int q0) {
    constexpr int P = kStageBytes / (HD * 2);
    constexpr int MT = P / 16 / kConsumerWarps;  // key tiles per warp per stage
    constexpr int KS = HD / 16;                  // k-steps of the score mma
    constexpr int DT = HD / 16;                  // dimension tiles of the P.V mma
    // full unrolling on the tensor-core kernel (an instance in the batch-1
    // kernel, which runs attn_ff, would unroll less to keep its registers)
    constexpr int KU = BATCHED ? KS : 2, DU = BATCHED ? DT : 4;
    constexpr uint32_t CBB = (uint32_t)P * 128u;  // bytes of one 64-column block of a stage
    const int gq = lane >> 2, cq = lane & 3;
    // The tensor-core kernel rounds q and the probabilities to one bf16, like
    // its GEMV inputs.  SPLIT (not taken: the batch-1 kernel runs attn_ff)
    // would take them as sums of two bf16 parts (hi + lo), whose two mma keep
    // scores and outputs at about fp32 accuracy (keys and values are bf16 already).
    constexpr bool SPLIT = !BATCHED;
    uint32_t qf[KS][2], ql[KS][2];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      if (gq < G) {
        const float* qh = ctl->qs + gq * HD + ks * 16 + 2 * cq;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float x0 = qh[8 * h], x1 = qh[8 * h + 1];
          const uint32_t hi = pack_bf16x2(x0, x1);
          qf[ks][h] = hi;
          ql[ks][h] = SPLIT ? pack_bf16x2(x0 - bf16_lo(hi), x1 - bf16_hi(hi)) : 0u;
        }
      } else {
        qf[ks][0] = qf[ks][1] = ql[ks][0] = ql[ks][1] = 0u;
      }
    }
    float o[DT][4];
#pragma unroll
    for (int dt = 0; dt < DT; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    float m0 = -1e30f, m1 = -1e30f, l0 = 0.f, l1 = 0.f;  // heads 2cq and 2cq + 1
    const uint32_t r7 = (uint32_t)(lane & 7);
    // ldmatrix rows: K tile row (lane & 15); V tile row (lane & 7) + 8 (lane >> 4)
    const uint32_t krow = (uint32_t)(lane & 15) * 128u;
    const uint32_t vrow = (uint32_t)((lane & 7) + ((lane >> 4) << 3)) * 128u;
    for (int s = 0; s < a.nsub; ++s) {
      const int np = min(P, a.n_cached - s * P);
      const uint32_t Ks = smem_addr(wait_stage(k));
      uint8_t* Vp = const_cast<uint8_t*>(wait_stage(k + 1));
      const uint32_t Vs = smem_addr(Vp);
      if (tr && s == 0) tr[5] = globaltimer();
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int key0 = (warp * MT + mt) * 16;
        if (key0 < np) {
          float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll KU
          for (int ks = 0; ks < KS; ++ks) {
            const uint32_t ch = ((uint32_t)(ks & 3) << 1) | (uint32_t)(lane >> 4);
            uint32_t af[4];
            ldmatrix_x4(af, Ks + (uint32_t)(ks >> 2) * CBB + (uint32_t)key0 * 128u + krow + ((ch ^ r7) << 4));
            mma16816(sc, af[0], af[1], af[2], af[3], qf[ks][0], qf[ks][1]);
            if (SPLIT) mma16816(sc, af[0], af[1], af[2], af[3], ql[ks][0], ql[ks][1]);
          }
          // this lane: keys key0 + gq (sc[0..1]) and key0 + gq + 8 (sc[2..3]), heads 2cq, 2cq + 1
          const bool v0 = key0 + gq < np, v1 = key0 + gq + 8 < np;
          const float s00 = v0 ? sc[0] : -1e30f, s01 = v0 ? sc[1] : -1e30f;
          const float s10 = v1 ? sc[2] : -1e30f, s11 = v1 ? sc[3] : -1e30f;
          float x0 = fmaxf(s00, s10), x1 = fmaxf(s01, s11);
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
            x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
          }
          const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
          const float c0 = exp2f(m0 - n0), c1 = exp2f(m1 - n1);
          const float p00 = v0 ? exp2f(s00 - n0) : 0.f, p01 = v0 ? exp2f(s01 - n1) : 0.f;
          const float p10 = v1 ? exp2f(s10 - n0) : 0.f, p11 = v1 ? exp2f(s11 - n1) : 0.f;
          float y0 = p00 + p10, y1 = p01 + p11;
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            y0 += __shfl_xor_sync(0xffffffffu, y0, off);
            y1 += __shfl_xor_sync(0xffffffffu, y1, off);
          }
          l0 = l0 * c0 + y0;
          l1 = l1 * c1 + y1;
          m0 = n0;
          m1 = n1;
#pragma unroll DU
          for (int dt = 0; dt < DT; ++dt) {
            o[dt][0] *= c0;
            o[dt][1] *= c1;
            o[dt][2] *= c0;
            o[dt][3] *= c1;
          }
          // P[keys 2cq, 2cq+1][head gq] and P[keys 8+2cq, 9+2cq][head gq], each as hi + lo bf16
          const uint32_t ph0 = pack_bf16x2(p00, p01), ph1 = pack_bf16x2(p10, p11);
          const uint32_t pb0 = movmatrix_trans(ph0), pb1 = movmatrix_trans(ph1);
          const uint32_t pl0 = SPLIT ? movmatrix_trans(pack_bf16x2(p00 - bf16_lo(ph0), p01 - bf16_hi(ph0))) : 0u;
          const uint32_t pl1 = SPLIT ? movmatrix_trans(pack_bf16x2(p10 - bf16_lo(ph1), p11 - bf16_hi(ph1))) : 0u;
          if (key0 + 16 > np) {
            // V rows past the cached positions may hold anything (0 * NaN is
            // NaN): zero this tile's absent rows, in every 64-column block
            for (int idx = lane; idx < 16 * (HD / 8); idx += 32) {
              const int r = idx / (HD / 8), c16 = idx % (HD / 8);
              if (key0 + r >= np)
                *reinterpret_cast<uint4*>(Vp + (c16 >> 3) * CBB + (uint32_t)(key0 + r) * 128u + (c16 & 7) * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            // order the generic writes before the ring's next TMA write of this slot
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
          }
#pragma unroll DU
          for (int dt = 0; dt < DT; ++dt) {
            const uint32_t ch = ((uint32_t)(dt & 3) << 1) | (uint32_t)((lane >> 3) & 1);
            uint32_t af[4];
            ldmatrix_x4_trans(af, Vs + (uint32_t)(dt >> 2) * CBB + (uint32_t)key0 * 128u + vrow + ((ch ^ r7) << 4));
            mma16816(o[dt], af[0], af[1], af[2], af[3], pb0, pb1);
            if (SPLIT) mma16816(o[dt], af[0], af[1], af[2], af[3], pl0, pl1);
          }
        }
      }
      release();  // K slot
      release();  // V slot
    }
    if (tr) tr[6] = globaltimer();
    if (a.owns_new && warp == 0) {
      // the new token: score of head (lane & 7), four lanes per head over
      // interleaved dimensions, then folded into warp 0's running state
      const int h = lane & 7, part = lane >> 3;
      float d = 0.f;
      if (h < G) {
#pragma unroll 8
        for (int e = 0; e < HD / 4; ++e)
          d = fmaf(ctl->qs[h * HD + e * 4 + part], bf16_bits_to_f32(ctl->knew[e * 4 + part]), d);
      }
      d += __shfl_xor_sync(0xffffffffu, d, 8);
      d += __shfl_xor_sync(0xffffffffu, d, 16);
      const float sn0 = __shfl_sync(0xffffffffu, d, 2 * cq), sn1 = __shfl_sync(0xffffffffu, d, 2 * cq + 1);
      const float n0 = fmaxf(m0, sn0), n1 = fmaxf(m1, sn1);
      const float c0 = exp2f(m0 - n0), c1 = exp2f(m1 - n1);
      const float e0 = exp2f(sn0 - n0), e1 = exp2f(sn1 - n1);
      l0 = l0 * c0 + e0;
      l1 = l1 * c1 + e1;
      m0 = n0;
      m1 = n1;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        const float va = bf16_bits_to_f32(ctl->vnew[dt * 16 + gq]), vb = bf16_bits_to_f32(ctl->vnew[dt * 16 + gq + 8]);
        o[dt][0] = o[dt][0] * c0 + e0 * va;
        o[dt][1] = o[dt][1] * c1 + e1 * va;
        o[dt][2] = o[dt][2] * c0 + e0 * vb;
        o[dt][3] = o[dt][3] * c1 + e1 * vb;
      }
    }
    // -- merge the warps through shared memory, HR heads per round
    constexpr int HR = kRedFloats / (kConsumerWarps * HD) < G ? kRedFloats / (kConsumerWarps * HD) : G;
    const size_t pbase = ((size_t)a.b * p.nq + q0) * p.n_chunks + a.c;
    if (gq == 0) {
      ctl->aml[(warp * kMaxGroup + 2 * cq) * 2] = m0;
      ctl->aml[(warp * kMaxGroup + 2 * cq) * 2 + 1] = l0;
      ctl->aml[(warp * kMaxGroup + 2 * cq + 1) * 2] = m1;
      ctl->aml[(warp * kMaxGroup + 2 * cq + 1) * 2 + 1] = l1;
    }
#pragma unroll
    for (int h0 = 0; h0 < G; h0 += HR) {
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int hh = 2 * cq + (e & 1) - h0, dim = dt * 16 + gq + 8 * (e >> 1);
          if (hh >= 0 && hh < HR) red[(warp * HR + hh) * HD + dim] = o[dt][e];
        }
      }
      consumer_bar();
      for (int id = t; id < HR * HD; id += kConsumerThreads) {
        const int hh = id / HD, d = id % HD, h = h0 + hh;
        float M = -1e30f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, ctl->aml[(w * kMaxGroup + h) * 2]);
        float den = 0.f, num = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float c = exp2f(ctl->aml[(w * kMaxGroup + h) * 2] - M);
          den = fmaf(c, ctl->aml[(w * kMaxGroup + h) * 2 + 1], den);
          num = fmaf(c, red[(w * HR + hh) * HD + d], num);
        }
        if (a.npieces == 1) {  // the whole row: the output itself
          if constexpr (BATCHED)
            p.attn_bf[(size_t)a.b * p.nq * HD + (size_t)(q0 + h) * HD + d] = f32_to_bf16_bits(num / den);
          else
            p.attn[(size_t)a.b * p.nq * HD + (size_t)(q0 + h) * HD + d] = num / den;
        } else {
          const size_t pi = pbase + (size_t)h * p.n_chunks;
          p.part_o[pi * HD + d] = num;
          if (d == 0) {
            p.part_ml[pi * 2] = M;
            p.part_ml[pi * 2 + 1] = den;
          }
        }
      }
      consumer_bar();
    }
  }

  // One attention slot: this step's schedule gives the slot a run of units
  // (equal for every slot), cut into pieces at row boundaries.
  template <int HD, int G>
  __device__ __forceinline__ bool attn_run(const mk_instr& in, int layer, int sig_idx) {
    constexpr int NP = HD / 64;  // rotation pairs per lane
    // The schedule and the RoPE factors depend only on this step's lengths
    // and positions, not on its activations: fetch the first piece's before
    // the dependency wait.
    AttnSched sc;
    attn_sched(p, ctl, in, sc);
    const int j = in.a;
    const int64_t g0 = attn_slot_begin(sc, j), g1 = attn_slot_begin(sc, j + 1);
    int rb = -1;  // sequence whose RoPE factors csr holds
    float2 csr[NP];
    if (g0 < g1) {
      rb = attn_piece_at(sc, g0, j).b;
      const float2* cs = p.rope + (size_t)ctl->spos[rb] * (HD / 2);
#pragma unroll
      for (int q = 0; q < NP; ++q) csr[q] = __ldg(cs + lane + 32 * q);
    }
    if (!wait_counter(in.wait_idx, in.wait_count)) return false;
    if (tr) tr[1] = globaltimer();
    for (int64_t g = g0; g < g1;) {
      const AttnPiece pc = attn_piece_at(sc, g, j);
      g += pc.ub - pc.ua;
      if (pc.b != rb) {
        rb = pc.b;
        const float2* cs = p.rope + (size_t)ctl->spos[rb] * (HD / 2);
#pragma unroll
        for (int q = 0; q < NP; ++q) csr[q] = __ldg(cs + lane + 32 * q);
      }
      attn_piece<HD, G>(attn_geo(p, ctl, pc, layer, HD), layer, sig_idx, csr);
    }
    return true;
  }

  // One piece of (sequence, KV head, head group): q of the G query heads of
  // the group against the piece's cached K/V rows (streamed through the ring)
  // and, in the piece that holds it, the new token's own K/V row.  The result
  // is an unnormalised partial (o, m, l) in log2 units; the last piece of the
  // row to finish merges all partials.
  // csr: the RoPE factors (cos, sin) of this lane's rotation pairs at the
  // sequence's position.
  template <int HD, int G>
  __device__ __forceinline__ void attn_piece(const Attn& a, int layer, int sig_idx, const float2 (&csr)[HD / 64]) {
    constexpr int NP = HD / 64;    // rotation pairs per lane
    const int qd = p.nq * HD, kvd = p.nkv * HD;
    const float* qkv = p.qkv + (size_t)a.b * (qd + 2 * kvd);
    // G = query heads of this instruction: head group hg of KV head kvh
    const int group = p.nq / p.nkv, nhg = group / G;
    const int q0 = a.kvh * group + a.hg * G;  // first query head
    const float qscale = 1.4426950408889634f * rsqrtf((float)HD);  // log2(e) / sqrt(hd)
    if (a.active) {
      // -- prologue: q heads (qk-norm, RoPE, scale) and the new K/V row
      const int tasks = G + (a.owns_new ? 2 : 0);
      for (int task = warp; task < tasks; task += kConsumerWarps) {
        const bool is_v = task == G + 1;
        const float* src = task < G ? qkv + (q0 + task) * HD : qkv + qd + (is_v ? kvd : 0) + a.kvh * HD;
        float lo[NP], hi[NP];
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          lo[j] = __ldcg(src + lane + 32 * j);
          hi[j] = __ldcg(src + lane + 32 * j + HD / 2);
          ss += lo[j] * lo[j] + hi[j] * hi[j];
        }
        if (!is_v) {
          if (p.qk_norm) {
            ss = warp_sum(ss);
            const float sc = 1.f / sqrtf(ss / (float)HD + p.eps);
#pragma unroll
            for (int j = 0; j < NP; ++j) {
              const uint16_t* gn = task < G ? p.layers[layer].q_norm : p.layers[layer].k_norm;
              lo[j] = lo[j] * sc * bf16_bits_to_f32(gn[lane + 32 * j]);
              hi[j] = hi[j] * sc * bf16_bits_to_f32(gn[lane + 32 * j + HD / 2]);
            }
          }
#pragma unroll
          for (int j = 0; j < NP; ++j) {
            const float2 r = csr[j];
            const float x0 = lo[j], x1 = hi[j];
            lo[j] = x0 * r.x - x1 * r.y;
            hi[j] = x1 * r.x + x0 * r.y;
          }
        }
        if (task < G) {
#pragma unroll
          for (int j = 0; j < NP; ++j) {
            ctl->qs[task * HD + lane + 32 * j] = lo[j] * qscale;
            ctl->qs[task * HD + lane + 32 * j + HD / 2] = hi[j] * qscale;
          }
        } else {
          // the new row (bf16): kept for this instruction's own use, and
          // appended at index S by head group 0 (every group computes the
          // same bits)
          uint16_t* cache = (is_v ? p.vc : p.kc) + (size_t)kv_row(p, layer, a.b, a.kvh, a.S) * HD;
          uint16_t* keep = is_v ? ctl->vnew : ctl->knew;
#pragma unroll
          for (int j = 0; j < NP; ++j) {
            const uint16_t b0 = f32_to_bf16_bits(lo[j]), b1 = f32_to_bf16_bits(hi[j]);
            if (a.hg == 0) {
              cache[lane + 32 * j] = b0;
              cache[lane + 32 * j + HD / 2] = b1;
            }
            keep[lane + 32 * j] = b0;
            keep[lane + 32 * j + HD / 2] = b1;
          }
        }
      }
      consumer_bar();
      if (tr) tr[4] = globaltimer();
      if constexpr (BATCHED)
        attn_tc<HD, G>(a, q0);
      else
        attn_ff<HD, G>(a, q0);
    }
    if (a.npieces == 1) {  // written above: no partials to merge
      signal(sig_idx);
      return;
    }
    // -- ticket: the last piece of the row to arrive merges.  The barrier
    // orders every thread's partial stores before thread 0's acq_rel add at
    // gpu scope (cumulative), so the merging CTA's acquire sees them.
    consumer_bar();
    if (t == 0) {
      uint32_t* ticket = p.tickets + (((size_t)layer * p.B + a.b) * p.nkv + a.kvh) * nhg + a.hg;
      const uint32_t old = atom_acq_rel_add(ticket, 1u);
      const bool last = old + 1u == (uint32_t)a.npieces;
      // the row's pieces have all counted: ready for the next step
      if (last) *ticket = 0u;
      ctl->last = last;
    }
    consumer_bar();
    if (ctl->last) {
      // One round trip for the merge: the (m, l) of every (head, piece) go to
      // shared memory while each thread's output elements load the partial o
      // of their first kMergeAhead pieces into registers (the rest, for rows of
      // more pieces, load in the combine loop).
      constexpr int NOUT = (G * HD + kConsumerThreads - 1) / kConsumerThreads;
      constexpr int MA = kMergeAhead;
      const int nvalid = a.npieces;
      const size_t pg = ((size_t)a.b * p.nq + q0) * p.n_chunks;
      for (int idx = t; idx < G * nvalid; idx += kConsumerThreads) {
        const int h = idx / nvalid, c = idx % nvalid;
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml) + pg + (size_t)h * p.n_chunks + c);
        red[2 * idx] = ml.x;
        red[2 * idx + 1] = ml.y;
      }
      float po_r[NOUT][MA];
#pragma unroll
      for (int o = 0; o < NOUT; ++o) {
        const int idx = t + o * kConsumerThreads;
        const float* po = p.part_o + (pg + (size_t)(idx / HD) * p.n_chunks) * HD + idx % HD;
#pragma unroll
        for (int c = 0; c < MA; ++c) po_r[o][c] = idx < G * HD && c < nvalid ? __ldcg(po + (size_t)c * HD) : 0.f;
      }
      consumer_bar();
#pragma unroll
      for (int o = 0; o < NOUT; ++o) {
        const int idx = t + o * kConsumerThreads;
        if (idx < G * HD) {
          const int h = idx / HD, d = idx % HD;
          const float* ml = red + 2 * h * nvalid;
          float M = -1e30f;
          for (int c = 0; c < nvalid; ++c) M = fmaxf(M, ml[2 * c]);
          float den = 0.f, num = 0.f;
#pragma unroll
          for (int c = 0; c < MA; ++c) {
            if (c < nvalid) {
              const float w = exp2f(ml[2 * c] - M);
              den = fmaf(w, ml[2 * c + 1], den);
              num = fmaf(w, po_r[o][c], num);
            }
          }
          const float* po = p.part_o + (pg + (size_t)h * p.n_chunks) * HD + d;
#pragma unroll 8
          for (int c = MA; c < nvalid; ++c) {
            const float w = exp2f(ml[2 * c] - M);
            den = fmaf(w, ml[2 * c + 1], den);
            num = fmaf(w, __ldcg(po + (size_t)c * HD), num);
          }
          if constexpr (BATCHED)
            p.attn_bf[(size_t)a.b * qd + (size_t)(q0 + h) * HD + d] = f32_to_bf16_bits(num / den);
          else
            p.attn[(size_t)a.b * qd + (size_t)(q0 + h) * HD + d] = num / den;
        }
      }
      signal(sig_idx);
    }
  }

  __device__ __forceinline__ bool attn(const mk_instr& in, int layer, int sig_idx) {
    const int G = attn_heads_per_instr(p.nq / p.nkv);
    if (t == 0) ctl->xtag = 0u;  // the reduction buffer is about to be overwritten (ordered by the prologue's barrier)
    if (p.hd == 128) {
      switch (G) {
        case 1: return attn_run<128, 1>(in, layer, sig_idx);
        case 2: return attn_run<128, 2>(in, layer, sig_idx);
        default: return attn_run<128, 4>(in, layer, sig_idx);
      }
    }
    switch (G) {
      case 1: return attn_run<64, 1>(in, layer, sig_idx);
      case 2: return attn_run<64, 2>(in, layer, sig_idx);
      default: return attn_run<64, 4>(in, layer, sig_idx);
    }
  }
};

template <bool BATCHED>
__device__ __forceinline__ void run_consumers(const Params& p, const mk_instr* list, int n, Ctl* ctl, uint8_t* ring,
                                              float* red) {
  Consumer<BATCHED> cs(p, ctl, ring, red);
  uint64_t* trace = p.trace && threadIdx.x == 0 ? p.trace + (size_t)p.offsets[blockIdx.x] * kTraceStamps : nullptr;
  for (int i = 0; i < n; ++i) {
    const mk_instr in = list[i];
    const int op = op_of(in.op_layer), layer = layer_of(in.op_layer);
    cs.tr = trace ? trace + (size_t)i * kTraceStamps : nullptr;
    if (trace) trace[i * kTraceStamps + 0] = globaltimer();
    bool ok = true;
    switch (op) {
      case OP_EMBED:
        ok = cs.wait_counter(in.wait_idx, in.wait_count);
        if (ok) {
          if (trace) trace[i * kTraceStamps + 1] = globaltimer();
          cs.embed(in);
          if (trace) trace[i * kTraceStamps + 2] = globaltimer();
          cs.signal(in.sig_idx);
        }
        break;
      case OP_QKV:
      case OP_OPROJ:
      case OP_GATEUP:
      case OP_DOWN:
      case OP_LMHEAD:
      case OP_ROUTER:
      case OP_EXP_DOWN:
        ok = cs.gemv(in, op, layer);  // waits on the instruction's counter inside
        if (ok) {
          if (trace) trace[i * kTraceStamps + 2] = globaltimer();
          cs.signal(in.sig_idx);
        }
        break;
      case OP_EXP_GATEUP:
        ok = cs.moe_gateup(in, layer);
        if (ok) {
          if (trace) trace[i * kTraceStamps + 2] = globaltimer();
          cs.signal(in.sig_idx);
        }
        break;
      case OP_ATTN:
        ok = cs.attn(in, layer, in.sig_idx);
        if (trace) trace[i * kTraceStamps + 2] = globaltimer();
        break;
      default:
        ok = cs.wait_counter(in.wait_idx, in.wait_count);
        break;
    }
    if (!ok) {
      ctl->dead = 1;
      return;
    }
  }
}

template <bool BATCHED>
__global__ void __launch_bounds__(kThreads, 1) mk_persistent(const __grid_constant__ Params p) {
  using SM = Smem<BATCHED>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(smem + SM::kRing);
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + SM::kRing + SM::kRed);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SM::kNst; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], kConsumerWarps);
    }
    ctl->dead = 0;
    ctl->waiting = 0;
    ctl->last = 0;
    ctl->xtag = 0u;
    for (int b = 0; b < kMaxBatch; ++b) ctl->amax[b] = 0ull;
    ctl->moe_pub = 0;
    // a sticky error from an earlier step, or out-of-range inputs: do nothing
    int bad = ld_relaxed_i32(p.status) != 0;
    for (int b = 0; b < p.B && !bad; ++b) {
      const int S = p.seq_lens[b], pos = p.positions[b], tok = p.tokens[b];
      ctl->slen[b] = S;
      ctl->spos[b] = pos;
      if (S < 0 || S >= p.T || pos < 0 || pos >= p.T || tok < 0 || tok >= p.V) {
        set_status(p, MK_ERR_RANGE, b);
        bad = 1;
      }
      // paged cache: every page the step reads or writes is in the pool
      for (int j = 0; p.bt && !bad && j <= S / p.page; ++j) {
        const int pg = p.bt[(size_t)b * p.bt_stride + j];
        if (pg < 0 || pg >= p.n_pages) {
          set_status(p, MK_ERR_RANGE, b);
          bad = 1;
        }
      }
    }
    // the swizzled TMA boxes of the batched GEMV need 1024-byte aligned slots
    if (!bad && (smem_addr(ring) & 1023u) != 0) {
      set_status(p, MK_ERR_UNSUPPORTED, -3);
      bad = 1;
    }
    ctl->flag = bad;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (ctl->flag) return;

  const int n = p.offsets[blockIdx.x + 1] - p.offsets[blockIdx.x];
  const mk_instr* list = p.instrs + p.offsets[blockIdx.x];
  if (threadIdx.x >= kConsumerThreads) {
    if (threadIdx.x == kConsumerThreads) run_producer<BATCHED>(p, list, n, ctl, ring);
  } else {
    run_consumers<BATCHED>(p, list, n, ctl, ring, red);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t kernel_smem_bytes(bool batched) { return batched ? Smem<true>::kTotal : Smem<false>::kTotal; }

cudaError_t kernel_prepare() {
  cudaError_t e = cudaFuncSetAttribute(mk_persistent<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Smem<false>::kTotal);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(mk_persistent<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)Smem<true>::kTotal);
}

cudaError_t kernel_occupancy(int* blocks_per_sm, bool batched) {
  return batched ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, mk_persistent<true>, kThreads,
                                                                 Smem<true>::kTotal)
                 : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, mk_persistent<false>, kThreads,
                                                                 Smem<false>::kTotal);
}

cudaError_t launch_step(const Params& p, int n_blocks, cudaStream_t stream) {
  void* args[] = {const_cast<Params*>(&p)};
  if (p.tc)
    return cudaLaunchCooperativeKernel((const void*)mk_persistent<true>, dim3(n_blocks), dim3(kThreads), args,
                                       Smem<true>::kTotal, stream);
  return cudaLaunchCooperativeKernel((const void*)mk_persistent<false>, dim3(n_blocks), dim3(kThreads), args,
                                     Smem<false>::kTotal, stream);
}

}  // namespace mk
