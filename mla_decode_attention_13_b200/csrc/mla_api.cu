// Host side of the C ABI declared in include/mla_b200.h: argument checks,
// TMA tensor-map encoding, per-device launch geometry, and the launches.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <mutex>

#include "mla_layer.h"

#define MLA_API extern "C" __attribute__((visibility("default")))

namespace mla {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int pairs = 0;  // co-resident 2-CTA clusters of the decode kernel
  int sms = 0;
};

// Per-device launch geometry, looked up on the first call on a device (under
// g_mu) and read without the lock afterwards: g_dev_ready is published with
// release order after the fields are written.  The library assumes the
// device keeps its context for as long as the library is loaded.
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
std::atomic<bool> g_dev_ready[kMaxDevices];
std::atomic<PFN_cuTensorMapEncodeTiled_v12000> g_encode{nullptr};

int current_device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  if (g_dev_ready[dev].load(std::memory_order_acquire)) {
    *out = g_dev[dev];
    return MLA_OK;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!g_dev_ready[dev].load(std::memory_order_relaxed)) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (major != 10) return MLA_ERR_UNSUPPORTED;  // built for sm_100a only
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (decode_kernel_pairs(&d.pairs) != cudaSuccess) {
      cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    if (d.pairs < 1) return MLA_ERR_UNSUPPORTED;
    g_dev_ready[dev].store(true, std::memory_order_release);
  }
  *out = d;
  return MLA_OK;
}

int tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  PFN_cuTensorMapEncodeTiled_v12000 f = g_encode.load(std::memory_order_acquire);
  if (!f) {
    std::lock_guard<std::mutex> lock(g_mu);
    f = g_encode.load(std::memory_order_relaxed);
    if (!f) {
      void* ptr = nullptr;
      cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
      const cudaError_t e =
          cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || ptr == nullptr) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
      }
      f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
      g_encode.store(f, std::memory_order_release);
    }
  }
  *fn = f;
  return MLA_OK;
}

// Recently encoded tensor maps of this host thread, keyed by what they encode
// (which map, base address, rows).  A serving loop calls the decode with the
// same cache and a few rotating query buffers, so their maps are encoded once
// instead of on every call.  A map holds only the address and the layout, so
// it stays right for any later buffer at the same address and size.
enum MapKind : int {
  kMapK = 0,
  kMapV = 1,
  kMapQ = 2,
  kMapCodes = 3,
  kMapRope = 4,
  kMapVCodes = 5,
  kMapOut = 6,
  kMapKinds = 7
};

struct MapCache {
  static constexpr int kWays = 8;
  struct Entry {
    const void* base = nullptr;
    uint64_t rows = 0;
    CUtensorMap map;
  };
  Entry e[kMapKinds][kWays];
  int next[kMapKinds] = {};
};

thread_local MapCache t_maps;

template <typename EncodeFn>
int cached_map(int kind, const void* base, uint64_t rows, CUtensorMap* out, EncodeFn&& encode) {
  MapCache::Entry* ways = t_maps.e[kind];
  for (int k = 0; k < MapCache::kWays; ++k) {
    if (ways[k].base == base && ways[k].rows == rows) {
      *out = ways[k].map;
      return MLA_OK;
    }
  }
  const int st = encode(out);
  if (st != MLA_OK) return st;
  MapCache::Entry& slot = ways[t_maps.next[kind]];
  t_maps.next[kind] = (t_maps.next[kind] + 1) % MapCache::kWays;
  slot.base = base;
  slot.rows = rows;
  slot.map = *out;
  return MLA_OK;
}

// A [rows][576] bf16 row-major tensor viewed as (64 cols, rows, 9 panels)
// with strides (1152 B, 128 B): a box (64, box_rows, box_panels) lands in
// shared memory as box_panels panels of box_rows x 128 bytes, 128B-swizzled.
int encode_panels576(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, uint64_t rows,
                     uint32_t box_rows, uint32_t box_panels) {
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(kDqk / 64)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDqk) * 2, 128};
  const cuuint32_t box[3] = {64, box_rows, box_panels};
  const cuuint32_t elem[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// bf16 out [batch][R][512] as (512 cols, R rows, batch) with strides
// (1024 B, R * 1024 B): box (64, 32, 1) is 32 rows x 64 columns of one batch
// row's output, 128B-swizzled in shared memory (the decode kernel's bulk
// stores of its output tiles; rows past R fall outside the map).
int encode_out_rows(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, void* base, int R, int batch) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDv), static_cast<cuuint64_t>(R),
                              static_cast<cuuint64_t>(batch)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDv) * 2, static_cast<cuuint64_t>(R) * kDv * 2};
  const cuuint32_t box[3] = {64, 32, 1};
  const cuuint32_t elem[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// Scratch of mla_decode_noalloc: one fixed device array per GPU that loads
// the library (held until the process exits), shared by every call on that
// device.  In host code the name stands for a host-side shadow, not a device
// address, so the address is looked up per device with cudaGetSymbolAddress.
static_assert(MLA_NOALLOC_SCRATCH_BYTES % 16 == 0, "scratch size");
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call there; no allocation).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return MLA_OK;
}

// The cache as (64 cols, rows, 4 panels, 2 halves of 256 columns) with strides
// (1152 B, 128 B, 512 B): box (64, 64, 2, 2) at (0, y, 2c, 0) lands as the
// value tile of CTA c (columns [256h + 128c, +128) of 64 tokens, panels in
// [h][e] order, 128B-swizzled).
int encode_value_tiles(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, uint64_t rows) {
  const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(rows), 4, 2};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kDqk) * 2, 128, 512};
  const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(kPage), 2, 2};
  const cuuint32_t elem[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// FP8 cache: the latent codes [rows][512] u8 as (512 cols, rows), box (64
// codes, 64 tokens), unswizzled (64-byte rows in shared memory).
int encode_codes(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, uint64_t rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDv), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDv)};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kPage)};
  const cuuint32_t elem[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// FP8 cache: the latent codes as (128 cols, rows, 2 column blocks c, 2
// halves h) with strides (512 B, 128 B, 256 B): box (128, 64, 1, 2) at (0, y,
// c, 0) is CTA c's value columns [256h + 128c, +128) of 64 tokens, landing as
// [h][token][128 codes], unswizzled.
int encode_vcodes(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, uint64_t rows) {
  const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(rows), 2, 2};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kDv), 128, 256};
  const cuuint32_t box[4] = {128, static_cast<cuuint32_t>(kPage), 1, 2};
  const cuuint32_t elem[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// FP8 cache: the bf16 rope [rows][64] as (64 cols, rows), box (64, 64 tokens),
// 128B-swizzled: one page lands as a key panel's 64 rows.
int encode_rope(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, uint64_t rows) {
  const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kPage)};
  const cuuint32_t elem[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A [tokens][h_q][cols] bf16 tensor as (64 cols, tokens, cols / 64 panels,
// h_q) with strides (h_q * cols * 2 B, 128 B, cols * 2 B): box (64, box_rows,
// 2, 1) at (0, t0, z, h) lands as 2 panels of box_rows tokens x 128 bytes of
// head h, 128B-swizzled; tokens past the end read as zeros.
int encode_token_rows(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, uint64_t tokens,
                      int h_q, int cols, uint32_t box_rows) {
  const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(tokens), static_cast<cuuint64_t>(cols / 64),
                              static_cast<cuuint64_t>(h_q)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(h_q) * cols * 2, 128, static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[4] = {64, box_rows, 2, 1};
  const cuuint32_t elem[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// Per-head weights [h_q][512][128] bf16 as (64 cols, h_q * 512 rows, 2 panels)
// with strides (256 B, 128 B): box (64, box_rows, 2) lands as 2 panels of
// box_rows x 128 bytes, 128B-swizzled.
int encode_head_weights(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, int h_q,
                        uint32_t box_rows) {
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(h_q) * kDv, 2};
  const cuuint64_t strides[2] = {256, 128};
  const cuuint32_t box[3] = {64, box_rows, 2};
  const cuuint32_t elem[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// Shared argument checks and launch of mla_absorb_q / mla_up_project.
int projection_impl(const void* a, const void* extra, const void* w, int tokens, int h_q, void* out, bool absorb,
                    void* stream) {
  if (!a || !w || !out || (absorb && !extra)) return MLA_ERR_ARG;
  if (tokens < 1 || h_q < 1) return MLA_ERR_ARG;
  if (!aligned16(a) || !aligned16(w) || !aligned16(out) || (absorb && !aligned16(extra))) return MLA_ERR_ARG;
  // the grid's y dimension counts token tiles: at most 65535 of them
  if (h_q > kMaxHq || tokens > 65535 * (absorb ? kProjAbsorbTile : kProjUpTile)) return MLA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != MLA_OK) return st;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if ((st = tensor_map_encoder(&enc)) != MLA_OK) return st;
  ProjParams p;
  p.nb = proj_box_rows(tokens, absorb ? kProjAbsorbTile : kProjUpTile);
  if ((st = encode_token_rows(enc, &p.tm_a, a, static_cast<uint64_t>(tokens), h_q, absorb ? 128 : kDv,
                              static_cast<uint32_t>(p.nb))) != MLA_OK ||
      (st = encode_head_weights(enc, &p.tm_b, w, h_q, 128)) != MLA_OK)
    return st;
  p.w = w;
  p.extra = extra;
  p.out = out;
  p.tokens = tokens;
  p.h_q = h_q;
  if (launch_projection(p, absorb, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

bool shape_ok(int batch, int h_q, int s_q) {
  return batch >= 1 && h_q >= 1 && h_q <= kMaxHq && s_q >= 1 && s_q <= kMaxSq &&
         static_cast<long long>(batch) * s_q * h_q <= (1LL << 30);
}

// The cache of one call: a bf16 cache (kv), or an FP8 one (codes, rope, exps).
struct CacheRef {
  const void* kv = nullptr;
  const void* codes = nullptr;
  const void* rope = nullptr;
  const void* exps = nullptr;
  bool fp8() const { return kv == nullptr; }
  bool ok() const { return fp8() ? (codes && rope && exps && aligned16(codes) && aligned16(rope) && aligned16(exps))
                                 : aligned16(kv); }
};

int decode_impl(const void* q, const CacheRef& cache, int64_t num_pages, const int32_t* block_table,
                int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q, float softmax_scale,
                int causal, void* out, float* lse, void* metadata, void* workspace, size_t workspace_bytes,
                void* stream, void* ev_before, void* ev_after, int out_f32) {
  if (!q || !block_table || !seqlens || !out || !lse || !metadata) return MLA_ERR_ARG;
  if (!cache.ok()) return MLA_ERR_ARG;
  if (batch < 1 || h_q < 1 || s_q < 1 || max_pages_per_seq < 1 || num_pages < 1) return MLA_ERR_ARG;
  if (causal != 0 && causal != 1) return MLA_ERR_ARG;
  if (!std::isfinite(softmax_scale) || softmax_scale < 0.0f) return MLA_ERR_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(metadata)) return MLA_ERR_ARG;
  if (workspace && !aligned16(workspace)) return MLA_ERR_ARG;
  if (!shape_ok(batch, h_q, s_q)) return MLA_ERR_UNSUPPORTED;
  if (num_pages > (1LL << 25)) return MLA_ERR_UNSUPPORTED;  // row coordinates stay below 2^31

  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != MLA_OK) return st;
  const size_t need = workspace_bytes_for(dev.pairs, h_q, s_q);
  if (workspace_bytes < need || (need > 0 && workspace == nullptr)) return MLA_ERR_WORKSPACE;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if ((st = tensor_map_encoder(&enc)) != MLA_OK) return st;

  const int R = s_q * h_q;
  const int tr = tile_rows(h_q, s_q);
  const int slots = max_slots(dev.pairs);
  DecodeParams p = {};
  const uint64_t kv_rows = static_cast<uint64_t>(num_pages) * kPage;
  const uint64_t q_rows = static_cast<uint64_t>(batch) * R;
  if ((st = cached_map(kMapQ, q, q_rows, &p.tm_q,
                       [&](CUtensorMap* m) { return encode_panels576(enc, m, q, q_rows, kMTile / 2, kDqk / 64); })) !=
      MLA_OK)
    return st;
  p.fp8 = cache.fp8() ? 1 : 0;
  p.codes = static_cast<const uint8_t*>(cache.codes);
  p.exps = static_cast<const int8_t*>(cache.exps);
  if (cache.fp8()) {
    if ((st = cached_map(kMapCodes, cache.codes, kv_rows, &p.tm_codes,
                         [&](CUtensorMap* m) { return encode_codes(enc, m, cache.codes, kv_rows); })) != MLA_OK ||
        (st = cached_map(kMapRope, cache.rope, kv_rows, &p.tm_rope,
                         [&](CUtensorMap* m) { return encode_rope(enc, m, cache.rope, kv_rows); })) != MLA_OK ||
        (st = cached_map(kMapVCodes, cache.codes, kv_rows, &p.tm_vcodes,
                         [&](CUtensorMap* m) { return encode_vcodes(enc, m, cache.codes, kv_rows); })) != MLA_OK)
      return st;
  } else {
    const void* kv_cache = cache.kv;
    if ((st = cached_map(kMapK, kv_cache, kv_rows, &p.tm_k,
                         [&](CUtensorMap* m) { return encode_panels576(enc, m, kv_cache, kv_rows, kPage, 1); })) !=
            MLA_OK ||
        (st = cached_map(kMapV, kv_cache, kv_rows, &p.tm_v,
                         [&](CUtensorMap* m) { return encode_value_tiles(enc, m, kv_cache, kv_rows); })) != MLA_OK)
      return st;
  }
  if (!out_f32) {
    // keyed by (batch, R): the same buffer viewed with another row count is another map
    const uint64_t key = (static_cast<uint64_t>(batch) << 32) | static_cast<uint32_t>(R);
    if ((st = cached_map(kMapOut, out, key, &p.tm_out,
                         [&](CUtensorMap* m) { return encode_out_rows(enc, m, out, R, batch); })) != MLA_OK)
      return st;
  }
  p.block_table = block_table;
  p.seqlens = seqlens;
  p.out = out;
  p.lse = lse;
  p.o_part = static_cast<float*>(workspace);
  p.lse_part = workspace ? static_cast<float*>(workspace) + static_cast<size_t>(slots) * tr * kDv : nullptr;
  p.meta = static_cast<int32_t*>(metadata);
  p.num_pages = num_pages;
  p.max_pages = max_pages_per_seq;
  p.batch = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.R = R;
  p.n_mt = ceil_div(R, kMTile);
  p.causal = causal;
  p.tile_rows = tr;
  p.max_slots = slots;
  p.out_f32 = out_f32;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;

  CombineParams cp;
  cp.meta = static_cast<const int32_t*>(metadata);
  cp.o_part = p.o_part;
  cp.lse_part = p.lse_part;
  cp.out = out;
  cp.lse = lse;
  cp.batch = batch;
  cp.s_q = s_q;
  cp.h_q = h_q;
  cp.R = R;
  cp.tile_rows = tr;
  cp.pairs = dev.pairs;
  cp.max_slots = slots;
  cp.slices = combine_slices(batch * p.n_mt, tr, dev.sms);
  cp.out_f32 = out_f32;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Inside a stream capture the events must become event-record nodes of the
  // graph (external events), or they would never be recorded at replay.
  unsigned int ev_flags = cudaEventRecordDefault;
  if (ev_before || ev_after) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return MLA_ERR_CUDA;
    if (cs == cudaStreamCaptureStatusActive) ev_flags = cudaEventRecordExternal;
  }
  if (ev_before && cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev_before), s, ev_flags) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (launch_decode(p, dev.pairs, s) != cudaSuccess) return MLA_ERR_CUDA;
  if (ev_after && cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev_after), s, ev_flags) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (launch_combine(cp, 4 * dev.sms, s) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // namespace
}  // namespace mla

using namespace mla;

MLA_API size_t mla_metadata_bytes(int batch, int h_q, int s_q) {
  if (!shape_ok(batch, h_q, s_q)) return 0;
  return meta_layout(batch, h_q, s_q).words * sizeof(int32_t);
}

MLA_API size_t mla_workspace_bytes(int batch, int h_q, int s_q) {
  if (!shape_ok(batch, h_q, s_q)) return 0;
  DeviceInfo dev;
  if (current_device_info(&dev) != MLA_OK) return workspace_bytes_for(kMaxPairs, h_q, s_q);
  return workspace_bytes_for(dev.pairs, h_q, s_q);
}

MLA_API int mla_num_sm_pairs(void) {
  DeviceInfo dev;
  const int st = current_device_info(&dev);
  return st == MLA_OK ? dev.pairs : st;
}

MLA_API int mla_get_metadata(const int32_t* seqlens, int batch, int h_q, int s_q, void* metadata, void* stream) {
  if (!seqlens || !metadata) return MLA_ERR_ARG;
  if (batch < 1 || h_q < 1 || s_q < 1) return MLA_ERR_ARG;
  if (!aligned16(metadata)) return MLA_ERR_ARG;
  if (!shape_ok(batch, h_q, s_q)) return MLA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const int st = current_device_info(&dev);
  if (st != MLA_OK) return st;
  if (launch_sched(seqlens, batch, h_q, s_q, dev.pairs, static_cast<int32_t*>(metadata),
                   static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

MLA_API int mla_decode(const void* q, const void* kv_cache, int64_t num_pages, const int32_t* block_table,
                       int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q, float softmax_scale,
                       int causal, void* out, float* lse, void* metadata, void* workspace, size_t workspace_bytes,
                       void* stream) {
  CacheRef cache;
  cache.kv = kv_cache;
  return decode_impl(q, cache, num_pages, block_table, max_pages_per_seq, seqlens, batch, s_q, h_q, softmax_scale,
                     causal, out, lse, metadata, workspace, workspace_bytes, stream, nullptr, nullptr, 0);
}

MLA_API int mla_decode_f32(const void* q, const void* kv_cache, int64_t num_pages, const int32_t* block_table,
                           int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q,
                           float softmax_scale, int causal, float* out, float* lse, void* metadata, void* workspace,
                           size_t workspace_bytes, void* stream) {
  CacheRef cache;
  cache.kv = kv_cache;
  return decode_impl(q, cache, num_pages, block_table, max_pages_per_seq, seqlens, batch, s_q, h_q, softmax_scale,
                     causal, out, lse, metadata, workspace, workspace_bytes, stream, nullptr, nullptr, 1);
}

MLA_API int mla_decode_fp8(const void* q, const void* latent_codes, const void* rope, const int8_t* exps,
                           int64_t num_pages, const int32_t* block_table, int max_pages_per_seq, const int32_t* seqlens,
                           int batch, int s_q, int h_q, float softmax_scale, int causal, void* out, float* lse,
                           void* metadata, void* workspace, size_t workspace_bytes, void* stream) {
  if (!latent_codes || !rope || !exps) return MLA_ERR_ARG;
  CacheRef cache;
  cache.codes = latent_codes;
  cache.rope = rope;
  cache.exps = exps;
  return decode_impl(q, cache, num_pages, block_table, max_pages_per_seq, seqlens, batch, s_q, h_q, softmax_scale,
                     causal, out, lse, metadata, workspace, workspace_bytes, stream, nullptr, nullptr, 0);
}

MLA_API int mla_decode_fp8_timed(const void* q, const void* latent_codes, const void* rope, const int8_t* exps,
                                 int64_t num_pages, const int32_t* block_table, int max_pages_per_seq,
                                 const int32_t* seqlens, int batch, int s_q, int h_q, float softmax_scale, int causal,
                                 void* out, float* lse, void* metadata, void* workspace, size_t workspace_bytes,
                                 void* stream, void* event_before_decode, void* event_after_decode) {
  if (!latent_codes || !rope || !exps) return MLA_ERR_ARG;
  CacheRef cache;
  cache.codes = latent_codes;
  cache.rope = rope;
  cache.exps = exps;
  return decode_impl(q, cache, num_pages, block_table, max_pages_per_seq, seqlens, batch, s_q, h_q, softmax_scale,
                     causal, out, lse, metadata, workspace, workspace_bytes, stream, event_before_decode,
                     event_after_decode, 0);
}

MLA_API int mla_decode_timed(const void* q, const void* kv_cache, int64_t num_pages, const int32_t* block_table,
                             int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q,
                             float softmax_scale, int causal, void* out, float* lse, void* metadata, void* workspace,
                             size_t workspace_bytes, void* stream, void* event_before_decode,
                             void* event_after_decode) {
  CacheRef cache;
  cache.kv = kv_cache;
  return decode_impl(q, cache, num_pages, block_table, max_pages_per_seq, seqlens, batch, s_q, h_q, softmax_scale,
                     causal, out, lse, metadata, workspace, workspace_bytes, stream, event_before_decode,
                     event_after_decode, 0);
}

MLA_API int mla_decode_noalloc(const void* q, const void* kv_cache, int64_t num_pages, const int32_t* block_table,
                               int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q,
                               float softmax_scale, int causal, void* out, float* lse, void* metadata, void* stream) {
  if (!shape_ok(batch, h_q, s_q)) return batch < 1 || h_q < 1 || s_q < 1 ? MLA_ERR_ARG : MLA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != MLA_OK) return st;
  if (workspace_bytes_for(dev.pairs, h_q, s_q) > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_SCRATCH;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != MLA_OK) return st;
  CacheRef cache;
  cache.kv = kv_cache;
  return decode_impl(q, cache, num_pages, block_table, max_pages_per_seq, seqlens, batch, s_q, h_q, softmax_scale,
                     causal, out, lse, metadata, scratch, MLA_NOALLOC_SCRATCH_BYTES, stream, nullptr, nullptr, 0);
}

MLA_API int mla_absorb_q(const void* q_nope, const void* q_rope, const void* w_uk, int tokens, int h_q, void* q_out,
                         void* stream) {
  return projection_impl(q_nope, q_rope, w_uk, tokens, h_q, q_out, true, stream);
}

MLA_API int mla_up_project(const void* o_latent, const void* w_uv, int tokens, int h_q, void* o_out, void* stream) {
  return projection_impl(o_latent, nullptr, w_uv, tokens, h_q, o_out, false, stream);
}

namespace mla {
namespace {

int merge_impl(const void* outs, const float* lses, int splits, int batch, int s_q, int h_q, void* out, float* lse,
               void* stream, int in_f32) {
  if (!outs || !lses || !out || !lse) return MLA_ERR_ARG;
  if (splits < 1 || batch < 1 || s_q < 1 || h_q < 1) return MLA_ERR_ARG;
  if (!aligned16(outs) || !aligned16(out)) return MLA_ERR_ARG;
  if (!shape_ok(batch, h_q, s_q)) return MLA_ERR_UNSUPPORTED;
  if (static_cast<long long>(splits) * batch * s_q * h_q > (1LL << 31)) return MLA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const int st = current_device_info(&dev);
  if (st != MLA_OK) return st;
  MergeParams p;
  p.outs = outs;
  p.lses = lses;
  p.out = out;
  p.lse = lse;
  p.splits = splits;
  p.batch = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.in_f32 = in_f32;
  if (launch_merge(p, dev.sms, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

}  // namespace
}  // namespace mla

MLA_API int mla_merge_splits(const void* outs, const float* lses, int splits, int batch, int s_q, int h_q, void* out,
                             float* lse, void* stream) {
  return merge_impl(outs, lses, splits, batch, s_q, h_q, out, lse, stream, 0);
}

MLA_API int mla_merge_splits_f32(const float* outs, const float* lses, int splits, int batch, int s_q, int h_q,
                                 void* out, float* lse, void* stream) {
  return merge_impl(outs, lses, splits, batch, s_q, h_q, out, lse, stream, 1);
}

MLA_API int mla_selftest_bounded_wait(void* stream) {
  DeviceInfo dev;
  const int st = current_device_info(&dev);
  if (st != MLA_OK) return st;
  if (launch_wait_selftest(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

MLA_API int mla_check_device_error(const void* metadata, void* stream, uint32_t* error_word) {
  if (!metadata) return MLA_ERR_ARG;
  uint32_t word = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&word, static_cast<const int32_t*>(metadata) + kHError, sizeof(word), cudaMemcpyDeviceToHost,
                      s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  if (error_word) *error_word = word;
  return word == 0 ? MLA_OK : MLA_ERR_DEVICE;
}

MLA_API int mla_take_device_errors(void* stream, uint32_t* error_word) {
  uint32_t word = 0;
  uint32_t proj = 0;
  if (take_sticky_error(static_cast<cudaStream_t>(stream), &word) != cudaSuccess ||
      take_project_sticky_error(static_cast<cudaStream_t>(stream), &proj) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  word |= proj;
  if (error_word) *error_word = word;
  return word == 0 ? MLA_OK : MLA_ERR_DEVICE;
}

MLA_API const char* mla_error_string(int status) {
  switch (status) {
    case MLA_OK:
      return "ok";
    case MLA_ERR_ARG:
      return "invalid argument (null pointer, bad size or misaligned pointer)";
    case MLA_ERR_UNSUPPORTED:
      return "unsupported shape or device";
    case MLA_ERR_CUDA:
      return "CUDA runtime or driver call failed";
    case MLA_ERR_WORKSPACE:
      return "workspace smaller than mla_workspace_bytes()";
    case MLA_ERR_DEVICE:
      return "device error word set (see MLA_DEVERR_* bits)";
    case MLA_ERR_SCRATCH:
      return "shape needs more scratch than the fixed no-allocation buffer holds (use mla_decode with a workspace)";
    default:
      return "unknown status";
  }
}
