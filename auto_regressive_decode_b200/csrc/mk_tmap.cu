// TMA tensor maps of the weight matrices and KV caches.
//
// A row-major bf16 matrix W[N][K] (K a multiple of 64) is described as the
// 3-D tensor (64, N, K/64) with strides (2 B, 2K B, 128 B): element
// (c, r, kb) is W[r][64 kb + c].  A box of (64, kBBoxRows, kBChunk/64) then
// brings kBBoxRows rows of one kBChunk-column chunk into shared memory as
// [column block][row][64 columns], with the 128-byte swizzle (16-byte chunk
// c of 128-byte line L at position c ^ (L & 7)).  Coordinates past K/64 read
// as zeros (the tail chunk of a K that is not a multiple of kBChunk).  The KV
// caches get the same view with head_dim columns and one attention stage of
// positions per box.
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include <algorithm>

#include "mk_device.h"

namespace mk {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool encode_one(EncodeTiledFn enc, const void* w, int64_t rows, int K, uint8_t* out, int box_rows = kBBoxRows,
                int box_blocks = kBChunk / 64) {
  static_assert(sizeof(CUtensorMap) == 128, "tensor map size");
  if (!w || rows <= 0 || rows >= (1ll << 31) || K % 64) return false;  // rows are int coordinates
  CUtensorMap m;
  const cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(K / 64)};
  const cuuint64_t strides[2] = {(cuuint64_t)K * 2, 128};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)box_blocks};
  const cuuint32_t elem[3] = {1, 1, 1};
  const CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  memcpy(out, &m, sizeof(m));
  return true;
}

// Batch-1 row-stationary tiles: W[N][K] as the 2-D tensor (K, N) with row
// pitch 2K bytes, boxes of min(K, kB1Chunk) columns x box_rows rows, no
// swizzle: a box lands as [box_rows][box columns] bf16.  Columns past K read
// as zeros (the tail chunk of a K that is not a multiple of kB1Chunk).
bool encode_2d(EncodeTiledFn enc, const void* w, int64_t rows, int K, int box_rows, uint8_t* out) {
  if (!w || rows <= 0 || rows >= (1ll << 31) || K <= 0 || K % 8) return false;
  CUtensorMap m;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)(K < kB1Chunk ? K : kB1Chunk), (cuuint32_t)box_rows};
  const cuuint32_t elem[2] = {1, 1};
  const CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  memcpy(out, &m, sizeof(m));
  return true;
}

// The box maps of one matrix: 64, 32, 16, 8, 4, 2 and 1 rows (a height above the
// matrix's row count is encoded at that count; the kernel never uses it).
bool encode_set(EncodeTiledFn enc, const void* w, int64_t rows, int K, uint8_t* out) {
  for (int m = 0; m < kB1BoxHeights; ++m)
    if (!encode_2d(enc, w, rows, K, (int)std::min<int64_t>(kB1TallestBox >> m, rows), out + 128 * m)) return false;
  return true;
}

// Rows of head_dim elements in each KV cache (or page pool).
int64_t kv_cache_rows(const mk_model_desc& d, const mk_kv& kv) {
  return kv.block_table ? (int64_t)d.n_layers * kv.n_pages * d.n_kv_heads * kv.page_size
                        : (int64_t)d.n_layers * d.batch * d.n_kv_heads * d.max_ctx;
}

}  // namespace

cudaError_t encode_tmaps(const mk_model_desc& d, const mk_weights& w, const mk_kv& kv, uint8_t* out) {
  EncodeTiledFn enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  if (!batched(d)) {  // the batch-1 kernel's weight maps are encode_tmaps_b1's: here only the KV caches
    memset(out, 0, (size_t)(kTmapsPerLayer * d.n_layers + 3) * 128);
    uint8_t* g = out + (size_t)d.n_layers * kTmapsPerLayer * 128;
    const int64_t kv_rows = kv_cache_rows(d, kv);
    const int P = attn_stage_positions(d.head_dim);
    return encode_one(enc, kv.k, kv_rows, d.head_dim, g + 128, P, d.head_dim / 64) &&
                   encode_one(enc, kv.v, kv_rows, d.head_dim, g + 256, P, d.head_dim / 64)
               ? cudaSuccess
               : cudaErrorInvalidValue;
  }
  const int H = d.hidden, qd = d.n_q_heads * d.head_dim, kvd = d.n_kv_heads * d.head_dim;
  // MoE: the experts' matrices are stacked, [E][Ie][H] for gate and up and
  // [E][H][Ie] for down, and read as one tall matrix each
  const int E = d.n_experts, I = E ? d.expert_ffn_dim : d.ffn_dim;
  const int64_t gu_rows = E ? (int64_t)E * I : I, dn_rows = E ? (int64_t)E * H : H;
  memset(out, 0, (size_t)(kTmapsPerLayer * d.n_layers + 3) * 128);
  for (int l = 0; l < d.n_layers; ++l) {
    const mk_layer_weights& lw = w.layers[l];
    uint8_t* o = out + (size_t)l * kTmapsPerLayer * 128;
    const bool ok = encode_one(enc, lw.wq, qd, H, o) && encode_one(enc, lw.wk, kvd, H, o + 128) &&
                    encode_one(enc, lw.wv, kvd, H, o + 256) && encode_one(enc, lw.wo, H, qd, o + 384) &&
                    encode_one(enc, lw.w_gate, gu_rows, H, o + 512) && encode_one(enc, lw.w_up, gu_rows, H, o + 640) &&
                    encode_one(enc, lw.w_down, dn_rows, I, o + 768) && (!E || encode_one(enc, lw.router, E, H, o + 896));
    if (!ok) return cudaErrorInvalidValue;
  }
  const void* lm = d.tied_embeddings ? w.embed : w.lm_head;
  uint8_t* g = out + (size_t)d.n_layers * kTmapsPerLayer * 128;
  if (!encode_one(enc, lm, d.vocab, H, g)) return cudaErrorInvalidValue;
  // KV caches: rows are (layer, sequence, KV head, position), head_dim columns;
  // a box is one attention stage of positions
  const int64_t kv_rows = kv_cache_rows(d, kv);
  const int P = attn_stage_positions(d.head_dim);
  if (!encode_one(enc, kv.k, kv_rows, d.head_dim, g + 128, P, d.head_dim / 64) ||
      !encode_one(enc, kv.v, kv_rows, d.head_dim, g + 256, P, d.head_dim / 64))
    return cudaErrorInvalidValue;
  return cudaSuccess;
}

cudaError_t encode_tmaps_b1(const mk_model_desc& d, const mk_weights& w, uint8_t* out) {
  EncodeTiledFn enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  const int H = d.hidden, qd = d.n_q_heads * d.head_dim, kvd = d.n_kv_heads * d.head_dim, I = d.ffn_dim;
  memset(out, 0, n_tmaps_b1(d) * 128);
  for (int l = 0; l < d.n_layers; ++l) {
    const mk_layer_weights& lw = w.layers[l];
    uint8_t* o = out + (size_t)l * kB1MapsPerLayer * 128;
    const size_t m = 128 * kB1BoxHeights;  // bytes of one matrix's maps
    const bool ok = encode_set(enc, lw.wq, qd, H, o) && encode_set(enc, lw.wk, kvd, H, o + m) &&
                    encode_set(enc, lw.wv, kvd, H, o + 2 * m) && encode_set(enc, lw.wo, H, qd, o + 3 * m) &&
                    encode_set(enc, lw.w_gate, I, H, o + 4 * m) && encode_set(enc, lw.w_up, I, H, o + 5 * m) &&
                    encode_set(enc, lw.w_down, H, I, o + 6 * m);
    if (!ok) return cudaErrorInvalidValue;
  }
  const void* lm = d.tied_embeddings ? w.embed : w.lm_head;
  if (!encode_set(enc, lm, d.vocab, H, out + (size_t)d.n_layers * kB1MapsPerLayer * 128))
    return cudaErrorInvalidValue;
  return cudaSuccess;
}

}  // namespace mk
