// Host side of libdms: descriptor checks, the cache's memory plan inside the
// caller's buffer, the per-layer state machine and the launch sequence of each
// entry point.  No device memory is ever allocated here.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_map>
#include <utility>
#include <vector>

#include "dms_internal.cuh"

using namespace dms;

namespace {

constexpr int kMaxPrefillTokens = 1 << 18;
constexpr int kMaxSmsForWork = 160;  // bound used to size the decode work list
constexpr int kFuseDecideHeads = 64;  // decode decisions fused into the append up to B*Hkv heads

struct Plan {
  size_t ctrl, pos, count, carry, npages, page_table, slot_pos, ring, plan, kept, kept_count, kept_upto, scan, kept_k, kept_v, win_k,
      win_v, head_done, part_acc, part_ml, k_scale, v_scale, k_pool, v_pool, total;
  int maxp, cap, pre_pages, items_cap, first_free;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int elem_bytes(int dt) { return dt == DMS_F32 ? 4 : dt == DMS_BF16 ? 2 : 1; }

// Sources whose decision logit comes from a product of the hidden state with
// a weight table (the adapter with RMSNorm, and the importance score).
bool adapter_source(int src) { return src == DMS_ALPHA_PROJ || src == DMS_ALPHA_SCORE_LINEAR; }

int check_desc(const dms_cache_desc* d) {
  if (!d) return DMS_ERR_INVALID;
  if (d->num_layers <= 0 || d->batch <= 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0) return DMS_ERR_INVALID;
  if (d->head_dim != 64 && d->head_dim != 128) return DMS_ERR_INVALID;
  if (d->num_q_heads % d->num_kv_heads) return DMS_ERR_INVALID;
  if (d->num_q_heads / d->num_kv_heads > 16) return DMS_ERR_INVALID;
  if (d->block <= 0 || d->block % 16 || d->block > 4096) return DMS_ERR_INVALID;
  if (d->window <= d->block) return DMS_ERR_INVALID;  // block must be below the window
  if (d->max_positions <= 0 || d->max_positions > (1 << 20)) return DMS_ERR_INVALID;
  if (d->prealloc_tokens < 0 || d->pool_pages <= 0) return DMS_ERR_INVALID;
  if (d->act_dtype != DMS_F32 && d->act_dtype != DMS_BF16) return DMS_ERR_INVALID;
  if (!(d->kv_dtype == d->act_dtype || (d->kv_dtype == DMS_FP8_E4M3 && d->act_dtype == DMS_BF16)))
    return DMS_ERR_INVALID;
  if (d->alpha_per != DMS_ALPHA_PER_HEAD && d->alpha_per != DMS_ALPHA_PER_LAYER) return DMS_ERR_INVALID;
  if (d->alpha_source < DMS_ALPHA_PROJ || d->alpha_source > DMS_ALPHA_SCORE_LINEAR) return DMS_ERR_INVALID;
  if (adapter_source(d->alpha_source)) {
    if (d->hidden <= 0 || d->hidden % 8) return DMS_ERR_INVALID;
    if (d->num_kv_heads > 8 || static_cast<long>(d->num_kv_heads) * d->hidden > 40960) return DMS_ERR_INVALID;
  }
  if (!adapter_source(d->alpha_source) && d->num_kv_heads > 32) return DMS_ERR_INVALID;
  if (!(d->alpha_scale == d->alpha_scale) || !(d->rms_eps >= 0.0f)) return DMS_ERR_INVALID;
  if (d->decode_kernel < DMS_DECODE_AUTO || d->decode_kernel > DMS_DECODE_FLAT) return DMS_ERR_INVALID;
  if (d->decision_shift < -1 || d->decision_shift > 1) return DMS_ERR_INVALID;
  return DMS_OK;
}

Plan make_plan(const dms_cache_desc* d) {
  Plan p{};
  const size_t L = d->num_layers, B = d->batch, H = d->num_kv_heads, g = d->num_q_heads / d->num_kv_heads;
  p.maxp = (d->max_positions + d->block - 1) / d->block;
  p.cap = p.maxp * d->block;
  p.pre_pages = std::min(p.maxp, (d->prealloc_tokens + d->block - 1) / d->block);
  p.items_cap = static_cast<int>(std::max<size_t>(B * H * p.maxp, 4 * kMaxSmsForWork) + B * H);
  p.first_free = static_cast<int>(L * B * H * p.pre_pages);
  size_t o = 0;
  auto take = [&](size_t bytes, size_t al) {
    o = align_up(o, al);
    size_t r = o;
    o += bytes;
    return r;
  };
  p.ctrl = take(CTRL_WORDS * 4, 256);
  p.pos = take(L * B * 4, 256);
  p.count = take(L * B * H * 4, 256);
  p.carry = take(L * B * H * 4, 256);
  p.npages = take(L * B * H * 4, 256);
  p.page_table = take(L * B * H * p.maxp * 4, 256);
  p.slot_pos = take(L * B * H * p.cap * 4, 256);
  p.ring = take(L * B * H * d->window * 4, 256);
  p.plan = take(2 * L * B * H * 16, 256);
  p.kept = take(B * H * d->max_positions * 4, 256);
  p.kept_count = take(B * H * 4, 256);
  p.kept_upto = take(B * H * (d->max_positions + 1) * 4, 256);
  p.scan = take(B * H * static_cast<size_t>(prefill_scan_stride(d->max_positions, d->window)) * 4, 256);
  const size_t kept_rows_bytes = d->act_dtype == DMS_BF16 ? B * H * d->max_positions * d->head_dim * 2 : 0;
  p.kept_k = take(kept_rows_bytes, 1024);
  p.kept_v = take(kept_rows_bytes, 1024);
  const size_t win_rows_bytes = d->act_dtype == DMS_BF16 ? B * H * d->window * d->head_dim * 2 : 0;
  p.win_k = take(win_rows_bytes, 1024);
  p.win_v = take(win_rows_bytes, 1024);
  p.head_done = take(B * H * 4, 256);
  p.part_acc = take(static_cast<size_t>(p.items_cap) * g * d->head_dim * 4, 256);
  p.part_ml = take(static_cast<size_t>(p.items_cap) * g * 2 * 4, 256);
  p.k_scale = take(static_cast<size_t>(d->pool_pages) * 4, 256);
  p.v_scale = take(static_cast<size_t>(d->pool_pages) * 4, 256);
  const size_t page_bytes = static_cast<size_t>(d->block) * d->head_dim * elem_bytes(d->kv_dtype);
  p.k_pool = take(page_bytes * d->pool_pages, 1024);
  p.v_pool = take(page_bytes * d->pool_pages, 1024);
  p.total = align_up(o, 256);
  return p;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// Tensor map over a page pool viewed as a 2-D tensor [pool_pages * P rows, D].
// Boxes are `rows` rows by up to 128 bytes; bf16 tiles use the 128-byte
// swizzle; FP8 tiles none (widened in shared memory row by row), or with
// `fp8_lines` the 128-byte swizzle over 128-byte lines -- for D = 64 the
// pool viewed as [pool_pages * P / 2, 128] (two rows per line, boxes of
// rows / 2 lines) -- for ldmatrix straight from the codes.
bool make_pool_map(CUtensorMap* map, void* base, const dms_cache_desc* d, int rows, bool fp8_lines = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const int eb = elem_bytes(d->kv_dtype);
  const bool pair = fp8_lines && d->kv_dtype == DMS_FP8_E4M3 && d->head_dim == 64;
  const int width = pair ? 128 : d->head_dim;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(width),
                        static_cast<cuuint64_t>(d->pool_pages) * static_cast<cuuint64_t>(d->block) / (pair ? 2 : 1)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(width) * eb};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(std::min(width, 128 / eb)), static_cast<cuuint32_t>(pair ? rows / 2 : rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUtensorMapDataType dt = d->kv_dtype == DMS_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                           : d->kv_dtype == DMS_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                    : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (d->kv_dtype == DMS_FP8_E4M3) sw = fp8_lines ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = enc(map, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Generic bf16 tensor map with the 128-byte swizzle: dims/strides innermost
// first (strides in bytes for dims 1..rank-1).
bool make_bf16_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                   const cuuint32_t* box) {
  auto enc = tensor_map_encoder();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
  cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map of the adapter's hidden rows [B*T, hidden] for the tensor-core
// decision kernel (bf16 only); false when it cannot be built.
bool make_hidden_map(CUtensorMap* map, const dms_cache_desc* d, const void* hidden, int T) {
  if (d->act_dtype != DMS_BF16 || !hidden) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d->hidden), static_cast<cuuint64_t>(d->batch) * T};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d->hidden) * 2};
  const cuuint32_t box[2] = {64u, 64u};  // 64 hidden elements x 64 tokens
  return make_bf16_map(map, hidden, 2, dims, strides, box);
}

}  // namespace

// The last (cache, layer) this library enqueued work for on each stream
// (layer -1: every layer, e.g. a reset).  A decode kernel may read its
// layer's state before the previous kernel of the stream completes only when
// that kernel was for another (cache, layer).
namespace {
std::mutex g_track_mu;
std::unordered_map<cudaStream_t, std::pair<const void*, int>> g_last_launch;

bool track_launch(const void* cache, int layer, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_track_mu);
  auto it = g_last_launch.find(s);
  const bool other = it == g_last_launch.end() ||
                     !(it->second.first == cache && (it->second.second == layer || it->second.second < 0 || layer < 0));
  g_last_launch[s] = std::make_pair(cache, layer);
  return other;
}
void forget_cache(const void* cache) {
  std::lock_guard<std::mutex> lk(g_track_mu);
  for (auto it = g_last_launch.begin(); it != g_last_launch.end();)
    it = it->second.first == cache ? g_last_launch.erase(it) : std::next(it);
}
}  // namespace

struct dms_cache {
  dms_cache_desc desc;
  Plan plan;
  CacheView view;
  char* base;
  size_t bytes;
  int device;
  int num_sms;
  std::vector<int> positions;  // host copy of tokens appended per layer
  std::vector<char> prefilled;
  CUtensorMap kmap, vmap;      // pool pages, 16-row boxes
  CUtensorMap kmap32, vmap32;  // pool pages, 32-row boxes (flat decode kernel)
  CUtensorMap kmapc, vmapc;    // pool pages, the cluster decode kernel's boxes (FP8 swizzled)
  bool has_maps;
  CUtensorMap kept_kmap, kept_vmap;  // tcgen05 prefill: kept copies
  CUtensorMap win_kmap, win_vmap;    // tcgen05 prefill of a later chunk: window copies
  bool has_kept_maps = false;
  std::vector<char> decoded;  // a decode step ran on the layer since its last reset
  int compacted_layer = -1;  // layer whose kept list the prefill attention may use
  int compacted_len = 0;
  int compacted_pos0 = 0;    // position of that call's first token
  int worklist_layer = -1;   // layer whose decode work list is current
};

extern "C" {

void dms_cache_desc_default(dms_cache_desc* d) {
  if (!d) return;
  std::memset(d, 0, sizeof(*d));
  d->window = 512;
  d->block = 256;
  d->prealloc_tokens = 4096;
  d->act_dtype = DMS_BF16;
  d->kv_dtype = DMS_BF16;
  d->alpha_per = DMS_ALPHA_PER_HEAD;
  d->alpha_source = DMS_ALPHA_PROJ;
  d->alpha_scale = 100.0f;
  d->rms_eps = 1e-6f;
  d->disable_eviction = 0;
}

int dms_cache_bytes(const dms_cache_desc* desc, size_t* dev_bytes) {
  int e = check_desc(desc);
  if (e) return e;
  if (!dev_bytes) return DMS_ERR_INVALID;
  Plan p = make_plan(desc);
  if (static_cast<long long>(desc->pool_pages) < static_cast<long long>(p.first_free)) return DMS_ERR_INVALID;
  *dev_bytes = p.total;
  return DMS_OK;
}

int dms_cache_alloc(const dms_cache_desc* desc, void* dev_mem, size_t bytes, void* stream, dms_cache** out) {
  if (!out) return DMS_ERR_INVALID;
  *out = nullptr;
  int e = check_desc(desc);
  if (e) return e;
  Plan p = make_plan(desc);
  if (desc->pool_pages < p.first_free) return DMS_ERR_INVALID;
  if (!dev_mem || (reinterpret_cast<uintptr_t>(dev_mem) & 255)) return DMS_ERR_INVALID;
  if (bytes < p.total) return DMS_ERR_NOMEM;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, dev_mem) != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return DMS_ERR_INVALID;
  }
  dms_cache* c = new (std::nothrow) dms_cache();
  if (!c) return DMS_ERR_INVALID;
  c->desc = *desc;
  c->plan = p;
  c->base = static_cast<char*>(dev_mem);
  c->bytes = bytes;
  c->device = attr.device;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
    delete c;
    return DMS_ERR_CUDA;
  }
  c->positions.assign(desc->num_layers, 0);
  c->prefilled.assign(desc->num_layers, 0);
  c->decoded.assign(desc->num_layers, 0);
  CacheView& v = c->view;
  v.L = desc->num_layers;
  v.B = desc->batch;
  v.Hq = desc->num_q_heads;
  v.Hkv = desc->num_kv_heads;
  v.D = desc->head_dim;
  v.hidden = desc->hidden;
  v.w = desc->window;
  v.P = desc->block;
  v.maxp = p.maxp;
  v.cap = p.cap;
  v.pool_pages = desc->pool_pages;
  v.pre_pages = p.pre_pages;
  v.max_pos = desc->max_positions;
  v.kv_dtype = desc->kv_dtype;
  v.act_dtype = desc->act_dtype;
  v.alpha_per = desc->alpha_per;
  v.alpha_source = desc->alpha_source;
  v.disable = desc->disable_eviction ? 1 : 0;
  v.decode_kernel = desc->decode_kernel;
  v.shift = desc->decision_shift;
  v.alpha_scale = desc->alpha_scale;
  v.rms_eps = desc->rms_eps;
  v.num_sms = c->num_sms;
  char* b = c->base;
  v.ctrl = reinterpret_cast<int*>(b + p.ctrl);
  v.pos = reinterpret_cast<int*>(b + p.pos);
  v.count = reinterpret_cast<int*>(b + p.count);
  v.carry = reinterpret_cast<int*>(b + p.carry);
  v.npages = reinterpret_cast<int*>(b + p.npages);
  v.page_table = reinterpret_cast<int*>(b + p.page_table);
  v.slot_pos = reinterpret_cast<int*>(b + p.slot_pos);
  v.ring = reinterpret_cast<int*>(b + p.ring);
  v.plan = reinterpret_cast<int4*>(b + p.plan);
  v.kept = reinterpret_cast<int*>(b + p.kept);
  v.kept_count = reinterpret_cast<int*>(b + p.kept_count);
  v.kept_upto = reinterpret_cast<int*>(b + p.kept_upto);
  v.scan = reinterpret_cast<int*>(b + p.scan);
  v.scan_stride = prefill_scan_stride(desc->max_positions, desc->window);
  v.kept_k = desc->act_dtype == DMS_BF16 ? b + p.kept_k : nullptr;
  v.kept_v = desc->act_dtype == DMS_BF16 ? b + p.kept_v : nullptr;
  v.win_k = desc->act_dtype == DMS_BF16 ? b + p.win_k : nullptr;
  v.win_v = desc->act_dtype == DMS_BF16 ? b + p.win_v : nullptr;
  v.head_done = reinterpret_cast<int*>(b + p.head_done);
  v.part_acc = reinterpret_cast<float*>(b + p.part_acc);
  v.part_ml = reinterpret_cast<float*>(b + p.part_ml);
  v.items_cap = p.items_cap;
  v.k_scale = reinterpret_cast<float*>(b + p.k_scale);
  v.v_scale = reinterpret_cast<float*>(b + p.v_scale);
  v.k_pool = b + p.k_pool;
  v.v_pool = b + p.v_pool;
  c->has_maps = false;
  if (desc->kv_dtype != DMS_F32) {
    int prev = cur;
    if (prev != c->device) cudaSetDevice(c->device);
    const int crows = decode_cluster_box_rows(desc->head_dim, desc->kv_dtype == DMS_FP8_E4M3);
    c->has_maps = make_pool_map(&c->kmap, v.k_pool, desc, 16) && make_pool_map(&c->vmap, v.v_pool, desc, 16) &&
                  make_pool_map(&c->kmap32, v.k_pool, desc, 32) && make_pool_map(&c->vmap32, v.v_pool, desc, 32) &&
                  make_pool_map(&c->kmapc, v.k_pool, desc, crows, true) &&
                  make_pool_map(&c->vmapc, v.v_pool, desc, crows, true);
    if (prev != c->device) cudaSetDevice(prev);
    if (!c->has_maps) {
      delete c;
      return DMS_ERR_CUDA;
    }
  }
  if (desc->act_dtype == DMS_BF16) {
    const int D = desc->head_dim;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D),
                                static_cast<cuuint64_t>(desc->batch) * desc->num_kv_heads * desc->max_positions};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64u, 64u};  // 64-key tiles of the prefill attention
    const cuuint64_t wdims[2] = {static_cast<cuuint64_t>(D),
                                 static_cast<cuuint64_t>(desc->batch) * desc->num_kv_heads * desc->window};
    c->has_kept_maps = make_bf16_map(&c->kept_kmap, v.kept_k, 2, dims, strides, box) &&
                       make_bf16_map(&c->kept_vmap, v.kept_v, 2, dims, strides, box) &&
                       make_bf16_map(&c->win_kmap, v.win_k, 2, wdims, strides, box) &&
                       make_bf16_map(&c->win_vmap, v.win_v, 2, wdims, strides, box);
  }
  if (launch_init(v, true, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    delete c;
    return DMS_ERR_CUDA;
  }
  track_launch(c, -1, static_cast<cudaStream_t>(stream));
  *out = c;
  return DMS_OK;
}

int dms_cache_free(dms_cache* c) {
  forget_cache(c);
  delete c;
  return DMS_OK;
}

int dms_cache_reset(dms_cache* c, void* stream) {
  if (!c) return DMS_ERR_INVALID;
  track_launch(c, -1, static_cast<cudaStream_t>(stream));
  if (launch_init(c->view, false, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DMS_ERR_CUDA;
  std::fill(c->positions.begin(), c->positions.end(), 0);
  std::fill(c->prefilled.begin(), c->prefilled.end(), 0);
  std::fill(c->decoded.begin(), c->decoded.end(), 0);
  c->compacted_layer = -1;
  c->worklist_layer = -1;
  return DMS_OK;
}

int dms_cache_get_layout(const dms_cache* c, dms_cache_layout* l) {
  if (!c || !l) return DMS_ERR_INVALID;
  const Plan& p = c->plan;
  l->total_bytes = p.total;
  l->status = p.ctrl + CTRL_STATUS * 4;
  l->next_page = p.ctrl + CTRL_NEXT_PAGE * 4;
  l->pos = p.pos;
  l->count = p.count;
  l->npages = p.npages;
  l->page_table = p.page_table;
  l->slot_pos = p.slot_pos;
  l->ring = p.ring;
  l->k_pool = p.k_pool;
  l->v_pool = p.v_pool;
  l->k_scale = p.k_scale;
  l->v_scale = p.v_scale;
  l->max_pages_per_head = p.maxp;
  l->slot_capacity = p.cap;
  l->prealloc_pages = p.pre_pages;
  l->first_free_page = p.first_free;
  return DMS_OK;
}

int dms_cache_export(dms_cache* c, int layer, dms_cache_view* out, void* stream) {
  if (!c || !out || layer < 0 || layer >= c->desc.num_layers) return DMS_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const CacheView& v = c->view;
  const long nb = static_cast<long>(v.B) * v.Hkv, lbase = static_cast<long>(layer) * nb;
  // one plain copy per array (layer slices are contiguous)
  auto copy = [&](void* dst, const int* src, long n) -> bool {
    return !dst || cudaMemcpyAsync(dst, src, n * sizeof(int), cudaMemcpyDeviceToHost, s) == cudaSuccess;
  };
  const bool ok = copy(out->pos, v.pos + static_cast<long>(layer) * v.B, v.B) && copy(out->count, v.count + lbase, nb) &&
                  copy(out->npages, v.npages + lbase, nb) &&
                  copy(out->page_table, v.page_table + lbase * v.maxp, nb * v.maxp) &&
                  copy(out->slot_pos, v.slot_pos + lbase * v.cap, nb * v.cap) &&
                  copy(out->ring, v.ring + lbase * v.w, nb * v.w);
  if (!ok || cudaStreamSynchronize(s) != cudaSuccess) return DMS_ERR_CUDA;
  return DMS_OK;
}

int dms_cache_status(dms_cache* c, void* stream, int* status) {
  if (!c || !status) return DMS_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaMemcpyAsync(&h, c->view.ctrl + CTRL_STATUS, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DMS_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DMS_ERR_CUDA;
  *status = h;
  return DMS_OK;
}

int dms_cache_positions(const dms_cache* c, int layer) {
  if (!c || layer < 0 || layer >= c->desc.num_layers) return DMS_ERR_INVALID;
  return c->positions[layer];
}

static int check_decide(const dms_cache* c, const dms_decide_params* d) {
  if (!d || !d->offset) return DMS_ERR_INVALID;
  if (d->offset_batch_stride != 0 && d->offset_batch_stride != c->desc.num_kv_heads) return DMS_ERR_INVALID;
  if (adapter_source(c->desc.alpha_source)) {
    // the score source has no normalisation: norm_weight is not read
    const bool norm = c->desc.alpha_source == DMS_ALPHA_PROJ;
    if (!d->hidden || !d->proj_weight || (norm && !d->norm_weight)) return DMS_ERR_INVALID;
    const uintptr_t any = reinterpret_cast<uintptr_t>(d->hidden) |
                          (norm ? reinterpret_cast<uintptr_t>(d->norm_weight) : 0) |
                          reinterpret_cast<uintptr_t>(d->proj_weight);
    if (any & 15) return DMS_ERR_INVALID;  // read as 16-byte vectors
  }
  return DMS_OK;
}

static DecideArgs decide_args(const dms_cache* c, const dms_decide_params* d) {
  DecideArgs a{};
  a.hidden = d->hidden;
  a.gamma = c->desc.alpha_source == DMS_ALPHA_PROJ ? d->norm_weight : nullptr;  // none: ones
  a.W = d->proj_weight;
  a.bias = d->proj_bias;
  a.offset = d->offset;
  a.offset_bstride = d->offset_batch_stride;
  return a;
}

int dms_decide(dms_cache* c, int T, const dms_decide_params* d, void* neuron_src, float* alpha, void* stream) {
  if (!c || !alpha || T <= 0 || T > c->desc.max_positions) return DMS_ERR_INVALID;
  int e = check_decide(c, d);
  if (e) return e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t r;
  if (adapter_source(c->desc.alpha_source)) {
    CUtensorMap hm;
    const bool have = make_hidden_map(&hm, &c->desc, d->hidden, T);
    r = launch_decide_proj(c->view, T, decide_args(c, d), alpha, have ? &hm : nullptr, s);
  } else {
    if (!neuron_src) return DMS_ERR_INVALID;
    const bool key = c->desc.alpha_source == DMS_ALPHA_KEY_NEURON;
    r = launch_neuron_rope(c->view, T, nullptr, key ? nullptr : neuron_src, key ? neuron_src : nullptr, d->offset,
                           d->offset_batch_stride, true, alpha, nullptr, nullptr, s);
  }
  return r == cudaSuccess ? DMS_OK : DMS_ERR_CUDA;
}

// q, k, v and o rows are moved as 16-byte vectors (and by TMA): their base
// pointers must be 16-byte aligned.
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static void prefill_maps(const dms_cache* c, int T, const void* q, const void* k, const void* v, void* o,
                         PrefillMaps* out);

static int check_prefill(const dms_cache* c, int layer, const dms_prefill_args* a) {
  if (!c || !a || layer < 0 || layer >= c->desc.num_layers) return DMS_ERR_INVALID;
  const int T = a->seq_len;
  if (T <= 0 || T > c->desc.max_positions || T > kMaxPrefillTokens) return DMS_ERR_INVALID;
  if (!a->q || !a->k || !a->v || !a->o || !a->alpha) return DMS_ERR_INVALID;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o)) return DMS_ERR_INVALID;
  if ((a->rope_cos == nullptr) != (a->rope_sin == nullptr)) return DMS_ERR_INVALID;
  if (a->decide) return check_decide(c, a->decide);
  return DMS_OK;
}

// A later chunk of a chunked prefill (the layer already holds tokens) runs on
// the tcgen05 attention, which reads the window and kept copies: bf16
// activations and a GQA group that is a power of two up to 16.
static bool chunk_capable(const dms_cache* c) {
  const int g = c->desc.num_q_heads / c->desc.num_kv_heads;
  return c->has_kept_maps && g <= 16 && (g & (g - 1)) == 0;
}

int dms_prefill_compact(dms_cache* c, int layer, const dms_prefill_args* a, void* stream) {
  int e = check_prefill(c, layer, a);
  if (e) return e;
  // prefill-then-generate: prefills (chunks) may follow each other until the
  // layer's first decode step
  if (c->decoded[layer]) return DMS_ERR_STATE;
  const int T = a->seq_len, T0 = c->positions[layer];
  if (T0 + T > c->desc.max_positions) return DMS_ERR_INVALID;
  if (T0 > 0 && (!chunk_capable(c) || prefill_scan_smem(c->view, T0, T) > (200u << 10))) return DMS_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  track_launch(c, layer, s);
  const CacheView& v = c->view;
  const bool neuron = a->decide && !adapter_source(c->desc.alpha_source);
  if (a->decide && !neuron) {
    CUtensorMap hm;
    const bool have = make_hidden_map(&hm, &c->desc, a->decide->hidden, T);
    if (launch_decide_proj(v, T, decide_args(c, a->decide), a->alpha, have ? &hm : nullptr, s) != cudaSuccess)
      return DMS_ERR_CUDA;
  }
  if (neuron || a->rope_cos) {
    // a later chunk's tokens sit at positions T0 + t (read on the device)
    if (launch_neuron_rope(v, T, T0 > 0 ? v.pos + static_cast<long>(layer) * v.B : nullptr, a->q, a->k,
                           neuron ? a->decide->offset : nullptr, neuron ? a->decide->offset_batch_stride : 0, neuron,
                           a->alpha, a->rope_cos, a->rope_sin, s) != cudaSuccess)
      return DMS_ERR_CUDA;
  }
  if (T0 > 0 && launch_prefill_context(v, layer, T0, T, a->alpha, s) != cudaSuccess) return DMS_ERR_CUDA;
  if (launch_prefill_scan(v, layer, T0, T, a->alpha, s) != cudaSuccess) return DMS_ERR_CUDA;
  if (launch_prefill_scatter(v, layer, T0, T, a->k, a->v, s) != cudaSuccess) return DMS_ERR_CUDA;
  c->prefilled[layer] = 1;
  c->positions[layer] = T0 + T;
  c->compacted_layer = layer;
  c->compacted_len = T;
  c->compacted_pos0 = T0;
  return DMS_OK;
}

int dms_prefill_attention(dms_cache* c, int layer, const dms_prefill_args* a, void* stream) {
  int e = check_prefill(c, layer, a);
  if (e) return e;
  if (c->compacted_layer != layer || c->compacted_len != a->seq_len ||
      c->compacted_pos0 + a->seq_len != c->positions[layer] || c->decoded[layer])
    return DMS_ERR_STATE;
  const int T0 = c->compacted_pos0;
  track_launch(c, layer, static_cast<cudaStream_t>(stream));
  PrefillMaps maps{};
  prefill_maps(c, a->seq_len, a->q, a->k, a->v, a->o, &maps);
  if (T0 > 0 && !maps.valid) return DMS_ERR_INVALID;
  if (launch_prefill_attention(c->view, T0, a->seq_len, a->q, a->k, a->v, a->o, &maps,
                               static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DMS_ERR_CUDA;
  return DMS_OK;
}

// Tensor maps of one call's q, k, v, o for the tcgen05 attention (valid only
// for bf16 activations and a GQA group that is a power of two up to 16).
static void prefill_maps(const dms_cache* c, int T, const void* q, const void* k, const void* v, void* o,
                         PrefillMaps* out) {
  PrefillMaps& maps = *out;
  maps.valid = false;
  const int g = c->desc.num_q_heads / c->desc.num_kv_heads;
  if (c->has_kept_maps && g <= 16 && (g & (g - 1)) == 0) {
    const int D = c->desc.head_dim;
    const cuuint64_t bt = static_cast<cuuint64_t>(c->desc.batch) * T;
    const cuuint64_t qd[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(c->desc.num_q_heads), bt};
    const cuuint64_t qs[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(c->desc.num_q_heads) * D * 2};
    const cuuint32_t qb[3] = {64u, static_cast<cuuint32_t>(g), static_cast<cuuint32_t>(128 / g)};
    const cuuint64_t kd[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(c->desc.num_kv_heads), bt};
    const cuuint64_t ks[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(c->desc.num_kv_heads) * D * 2};
    const cuuint32_t kbx[3] = {64u, 1u, 64u};
    // o as [B][T][Hq][D] (rank 4, so rows at or past T are clipped from stores)
    const cuuint64_t od[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(c->desc.num_q_heads),
                              static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(c->desc.batch)};
    const cuuint64_t os[3] = {qs[0], qs[1], qs[1] * T};
    const cuuint32_t ob[4] = {64u, static_cast<cuuint32_t>(g), static_cast<cuuint32_t>(128 / g), 1u};
    maps.valid = make_bf16_map(&maps.q, q, 3, qd, qs, qb) && make_bf16_map(&maps.k, k, 3, kd, ks, kbx) &&
                 make_bf16_map(&maps.v, v, 3, kd, ks, kbx) && make_bf16_map(&maps.o, o, 4, od, os, ob);
    maps.kept_k = c->kept_kmap;
    maps.kept_v = c->kept_vmap;
    maps.win_k = c->win_kmap;
    maps.win_v = c->win_vmap;
  }
}

int dms_train_gate(dms_cache* c, int T, const float* alpha, const float* noise, float tau, float* prob, float* hard,
                   float* penalty, void* stream) {
  if (!c || !alpha || !prob || !hard || !penalty || T <= 0) return DMS_ERR_INVALID;
  if (!(tau > 0.0f) || !(tau < INFINITY)) return DMS_ERR_INVALID;
  if (launch_train_gate(static_cast<long>(c->desc.batch) * c->desc.num_kv_heads, T, alpha, noise, tau, prob, hard,
                        penalty, c->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DMS_ERR_CUDA;
  return DMS_OK;
}

int dms_train_attention(dms_cache* c, int T, const void* q, const void* k, const void* v, const float* penalty,
                        void* o, void* stream) {
  if (!c || !q || !k || !v || !o || !penalty || T <= 0) return DMS_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DMS_ERR_INVALID;
  PrefillMaps maps{};
  prefill_maps(c, T, q, k, v, o, &maps);
  if (!maps.valid) return DMS_ERR_INVALID;  // bf16 activations, g a power of two up to 16
  // the penalties as a [B*Hkv, T] fp32 tensor map (rows of 16-byte multiples)
  CUtensorMap pm;
  bool have_pm = false;
  if (T % 4 == 0 && (reinterpret_cast<uintptr_t>(penalty) & 15) == 0) {
    auto enc = tensor_map_encoder();
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(T),
                                static_cast<cuuint64_t>(c->desc.batch) * c->desc.num_kv_heads};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(T) * 4};
    const cuuint32_t box[2] = {64u, 1u}, estr[2] = {1u, 1u};
    have_pm = enc && enc(&pm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(penalty), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  track_launch(c, -1, static_cast<cudaStream_t>(stream));
  if (launch_prefill_attention_tc(c->view, 0, T, o, maps, static_cast<cudaStream_t>(stream), penalty,
                                  have_pm ? &pm : nullptr) != cudaSuccess)
    return DMS_ERR_CUDA;
  return DMS_OK;
}

int dms_prefill(dms_cache* c, int layer, const dms_prefill_args* a, void* stream) {
  int e = dms_prefill_compact(c, layer, a, stream);
  if (e) return e;
  return dms_prefill_attention(c, layer, a, stream);
}

int dms_decode_append(dms_cache* c, int layer, const dms_decode_args* a, void* stream) {
  if (!c || !a || layer < 0 || layer >= c->desc.num_layers) return DMS_ERR_INVALID;
  if (!a->q || !a->k || !a->v || !a->alpha) return DMS_ERR_INVALID;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v)) return DMS_ERR_INVALID;
  if ((a->rope_cos == nullptr) != (a->rope_sin == nullptr)) return DMS_ERR_INVALID;
  if (a->decide) {
    int e = check_decide(c, a->decide);
    if (e) return e;
  }
  if (!c->prefilled[layer] || c->positions[layer] >= c->desc.max_positions) return DMS_ERR_STATE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  track_launch(c, layer, s);
  const CacheView& v = c->view;
  const bool neuron = a->decide && !adapter_source(c->desc.alpha_source);
  // The adapter's decision logits are computed inside the append kernel when
  // the batch has few heads (one warp per dot product); otherwise by their own
  // kernel with one CTA per (head, sequence).
  const bool fuse = a->decide && !neuron && c->desc.batch * c->desc.num_kv_heads <= kFuseDecideHeads;
  DecideArgs da{};
  if (a->decide && !neuron) {
    da = decide_args(c, a->decide);
    if (!fuse && launch_decide_proj(v, 1, da, a->alpha, nullptr, s) != cudaSuccess) return DMS_ERR_CUDA;
  }
  if (neuron || a->rope_cos) {
    // the token's position is read on the device from the layer's position counter
    if (launch_neuron_rope(v, 1, v.pos + static_cast<long>(layer) * v.B, a->q, a->k,
                           neuron ? a->decide->offset : nullptr, neuron ? a->decide->offset_batch_stride : 0, neuron,
                           a->alpha, a->rope_cos, a->rope_sin, s) != cudaSuccess)
      return DMS_ERR_CUDA;
  }
  if (launch_decode_append(v, layer, a->k, a->v, a->alpha, fuse ? &da : nullptr, c->num_sms, s) != cudaSuccess)
    return DMS_ERR_CUDA;
  c->decoded[layer] = 1;
  c->positions[layer] += 1;
  c->worklist_layer = layer;
  return DMS_OK;
}

}  // extern "C"

namespace {

// Decode attention over a layer's pages (fused: the whole decode step) with
// the kernel the descriptor selects; the flat kernel hands shapes it does not
// stage to the cluster kernel.
// after_wait: the previous kernel on the stream is a programmatic dependent
// that waited for everything before it (the rotary pass), so the layer's
// state may be read before this launch's own wait.
int run_decode_kernel(dms_cache* c, int layer, const void* q, void* o, bool fused, const void* k, const void* v,
                      float* alpha, const DecideArgs* da, cudaStream_t s, bool after_wait = false) {
  const CacheView& cv = c->view;
  const bool early = track_launch(c, layer, s) || after_wait;
  int mode = c->desc.decode_kernel;
  if (mode == DMS_DECODE_AUTO) mode = DMS_DECODE_CLUSTER;
  if (mode == DMS_DECODE_FLAT) {
    bool taken = false;
    if (launch_decode_flat(cv, layer, q, o, fused, k, v, alpha, da, &c->kmap32, &c->vmap32, s, early, &taken) !=
        cudaSuccess)
      return DMS_ERR_CUDA;
    if (taken) return DMS_OK;
  }
  return launch_decode_cluster(cv, layer, q, o, fused, k, v, alpha, da, &c->kmapc, &c->vmapc, c->num_sms, s, early) ==
                 cudaSuccess
             ? DMS_OK
             : DMS_ERR_CUDA;
}

}  // namespace

extern "C" {

int dms_decode_attention(dms_cache* c, int layer, const void* q, void* o, void* stream) {
  if (!c || !q || !o || layer < 0 || layer >= c->desc.num_layers) return DMS_ERR_INVALID;
  if (!aligned16(q) || !aligned16(o)) return DMS_ERR_INVALID;
  if (c->worklist_layer != layer) return DMS_ERR_STATE;
  if (c->has_maps && c->desc.kv_dtype != DMS_F32)
    return run_decode_kernel(c, layer, q, o, false, nullptr, nullptr, nullptr, nullptr,
                             static_cast<cudaStream_t>(stream));
  track_launch(c, layer, static_cast<cudaStream_t>(stream));
  if (launch_decode_attention(c->view, layer, q, o, c->has_maps ? &c->kmap : nullptr, c->has_maps ? &c->vmap : nullptr,
                              c->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DMS_ERR_CUDA;
  return DMS_OK;
}

int dms_decode_step(dms_cache* c, int layer, const dms_decode_args* a, void* stream) {
  if (!c || !a || !a->o || !aligned16(a->o)) return DMS_ERR_INVALID;
  if (c->desc.kv_dtype == DMS_F32) {
    int e = dms_decode_append(c, layer, a, stream);
    if (e) return e;
    return dms_decode_attention(c, layer, a->q, a->o, stream);
  }
  if (c->desc.kv_dtype == DMS_FP8_E4M3 && (c->desc.decode_kernel == DMS_DECODE_FLAT || !c->has_maps)) {
    // FP8 pages may be re-encoded by the append, so the attention follows it;
    // the flat kernel has no append-first step: the append kernel, then the
    // attention over the updated pages.  (The cluster kernel appends first
    // in the same launch.)
    int e = dms_decode_append(c, layer, a, stream);
    if (e) return e;
    return run_decode_kernel(c, layer, a->q, a->o, false, nullptr, nullptr, nullptr, nullptr,
                             static_cast<cudaStream_t>(stream));
  }
  if (layer < 0 || layer >= c->desc.num_layers) return DMS_ERR_INVALID;
  if (!a->q || !a->k || !a->v || !a->alpha) return DMS_ERR_INVALID;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v)) return DMS_ERR_INVALID;
  if ((a->rope_cos == nullptr) != (a->rope_sin == nullptr)) return DMS_ERR_INVALID;
  if (a->decide) {
    int e = check_decide(c, a->decide);
    if (e) return e;
  }
  if (!c->prefilled[layer] || c->positions[layer] >= c->desc.max_positions) return DMS_ERR_STATE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const CacheView& v = c->view;
  const bool neuron = a->decide && !adapter_source(c->desc.alpha_source);
  const bool rope = neuron || a->rope_cos;
  if (rope) {
    // the decision neuron / rotary pass, a programmatic dependent of the
    // previous kernel: it waits for it, then lets the step's launch read the
    // layer's state and request its first tiles while it runs
    track_launch(c, layer, s);
    if (launch_neuron_rope(v, 1, v.pos + static_cast<long>(layer) * v.B, a->q, a->k,
                           neuron ? a->decide->offset : nullptr, neuron ? a->decide->offset_batch_stride : 0, neuron,
                           a->alpha, a->rope_cos, a->rope_sin, s, true) != cudaSuccess)
      return DMS_ERR_CUDA;
  }
  DecideArgs da{};
  const bool proj = a->decide && !neuron;
  if (proj) da = decide_args(c, a->decide);
  // One launch -- bf16 pages: attention over the pre-append slots plus the new
  // token, then the append; FP8 pages: the append, then the attention over
  // the updated pages; with the adapter's decision logits computed inside.
  if (int e = run_decode_kernel(c, layer, a->q, a->o, true, a->k, a->v, a->alpha, proj ? &da : nullptr, s, rope))
    return e;
  c->decoded[layer] = 1;
  c->positions[layer] += 1;
  c->worklist_layer = layer;
  return DMS_OK;
}

int dms_decode_step_layers(dms_cache* c, int layer0, int num_layers, const dms_decode_args* a, void* stream) {
  if (!c || !a || num_layers < 1 || layer0 < 0 || layer0 + num_layers > c->desc.num_layers) return DMS_ERR_INVALID;
  if (!a->q || !a->k || !a->v || !a->o || !a->alpha) return DMS_ERR_INVALID;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o)) return DMS_ERR_INVALID;
  if ((a->rope_cos == nullptr) != (a->rope_sin == nullptr)) return DMS_ERR_INVALID;
  // one fused launch of the cluster kernel over the layers (bf16 or FP8 pages)
  if (c->desc.kv_dtype == DMS_F32 || !c->has_maps) return DMS_ERR_INVALID;
  if (a->decide) {
    int e = check_decide(c, a->decide);
    if (e) return e;
  }
  const int t = c->positions[layer0];
  for (int l = layer0; l < layer0 + num_layers; ++l)
    if (!c->prefilled[l] || c->positions[l] != t || t >= c->desc.max_positions) return DMS_ERR_STATE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const CacheView& v = c->view;
  const int B = c->desc.batch, Hq = c->desc.num_q_heads, Hkv = c->desc.num_kv_heads, D = c->desc.head_dim;
  const bool neuron = a->decide && !adapter_source(c->desc.alpha_source);
  const long ostride_layer = a->decide ? static_cast<long>(a->decide->offset_batch_stride ? B * Hkv : Hkv) : 0;
  const bool rope = neuron || a->rope_cos;
  if (rope) {
    // the decision neuron / rotary pass of each layer (its rows of q and k),
    // each a programmatic dependent of the kernel before it
    track_launch(c, -1, s);
    for (int l = 0; l < num_layers; ++l) {
      char* ql = static_cast<char*>(a->q) + static_cast<long>(l) * B * Hq * D * 2;
      char* kl = static_cast<char*>(a->k) + static_cast<long>(l) * B * Hkv * D * 2;
      if (launch_neuron_rope(v, 1, v.pos + static_cast<long>(layer0 + l) * B, ql, kl,
                             neuron ? a->decide->offset + l * ostride_layer : nullptr,
                             neuron ? a->decide->offset_batch_stride : 0, neuron, a->alpha + static_cast<long>(l) * B * Hkv,
                             a->rope_cos, a->rope_sin, s, true) != cudaSuccess)
        return DMS_ERR_CUDA;
    }
  }
  DecideArgs da{};
  const bool proj = a->decide && !neuron;
  if (proj) {
    da = decide_args(c, a->decide);
    da.gamma_lstride = c->desc.hidden;
    da.w_lstride = static_cast<long>(Hkv) * c->desc.hidden;
    da.bias_lstride = Hkv;
    da.offset_lstride = ostride_layer;
  }
  // every layer of the range in one launch (early reads only after the wait)
  track_launch(c, -1, s);
  if (launch_decode_cluster(v, layer0, a->q, a->o, true, a->k, a->v, a->alpha, proj ? &da : nullptr, &c->kmapc,
                            &c->vmapc, c->num_sms, s, false, num_layers) != cudaSuccess)
    return DMS_ERR_CUDA;
  for (int l = layer0; l < layer0 + num_layers; ++l) {
    c->decoded[l] = 1;
    c->positions[l] += 1;
  }
  c->worklist_layer = -1;
  return DMS_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Self-check of the failure path of a bounded device wait: one thread waits,
// with the library's bounded wait, on a shared-memory barrier that nothing
// completes (no copy or arrival is ever issued for it), gives up after `tries`
// tries and records DMS_ST_TIMEOUT in the cache's status word, exactly as a
// kernel whose copy never lands does.  Nothing is in flight when it returns.
// ---------------------------------------------------------------------------
namespace {
__global__ void k_wait_selftest(int* ctrl, long long tries) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, tries)) set_status(ctrl, DMS_ST_TIMEOUT);
}
}  // namespace

extern "C" int dms_selftest_wait_timeout(dms_cache* c, int tries, void* stream) {
  if (!c || tries <= 0 || tries > (1 << 24)) return DMS_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  track_launch(c, -1, s);
  k_wait_selftest<<<1, 32, 0, s>>>(c->view.ctrl, tries);
  return cudaGetLastError() == cudaSuccess ? DMS_OK : DMS_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Decode attention with its split-K partials in a fixed device array owned by
// the library, for callers that cannot provide scratch memory.  Nothing here
// allocates: the array is a file-scope __device__ variable, and its device
// address is looked up once per device.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB per device
static __device__ __align__(256) unsigned char g_split_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_split_scratch_addr[kMaxDevices] = {};

// Device address of g_split_scratch on `device`.  In host code the symbol is
// only a host-side stand-in; the real address comes from cudaGetSymbolAddress
// with that device current.  The lookup runs once per device, under a lock.
int split_scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return DMS_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_split_scratch_addr[device]) {
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) return DMS_ERR_CUDA;
    if (prev != device && cudaSetDevice(device) != cudaSuccess) return DMS_ERR_CUDA;
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_split_scratch);
    if (prev != device && cudaSetDevice(prev) != cudaSuccess) return DMS_ERR_CUDA;
    if (e != cudaSuccess || p == nullptr) return DMS_ERR_CUDA;
    g_split_scratch_addr[device] = p;
  }
  *out = g_split_scratch_addr[device];
  return DMS_OK;
}

}  // namespace

extern "C" int dms_decode_attention_noalloc(dms_cache* c, int layer, const void* q, void* o, void* stream) {
  if (!c || !q || !o || layer < 0 || layer >= c->desc.num_layers) return DMS_ERR_INVALID;
  if (!aligned16(q) || !aligned16(o)) return DMS_ERR_INVALID;
  if (c->worklist_layer != layer) return DMS_ERR_STATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c->desc.kv_dtype == DMS_F32) {
    // fp32 pages: one CTA per query head, no split-K partials, no scratch
    track_launch(c, layer, st);
    return launch_decode_attention(c->view, layer, q, o, nullptr, nullptr, c->num_sms, st) == cudaSuccess
               ? DMS_OK
               : DMS_ERR_CUDA;
  }
  const size_t g = static_cast<size_t>(c->desc.num_q_heads / c->desc.num_kv_heads);
  const size_t items = static_cast<size_t>(c->plan.items_cap);
  const size_t heads = static_cast<size_t>(c->desc.batch) * c->desc.num_kv_heads;
  const size_t cnt_bytes = align_up(heads * sizeof(int), 256);
  const size_t acc_bytes = align_up(items * g * c->desc.head_dim * sizeof(float), 256);
  const size_t ml_bytes = items * g * 2 * sizeof(float);
  if (cnt_bytes + acc_bytes + ml_bytes > kNoAllocScratchBytes) return DMS_ERR_SCRATCH_LIMIT;
  void* base = nullptr;
  const int e = split_scratch_address(c->device, &base);
  if (e) return e;
  unsigned char* p = static_cast<unsigned char*>(base);
  CacheView v = c->view;
  v.head_done = reinterpret_cast<int*>(p);  // per-head arrival counters: must start at zero
  v.part_acc = reinterpret_cast<float*>(p + cnt_bytes);
  v.part_ml = reinterpret_cast<float*>(p + cnt_bytes + acc_bytes);
  track_launch(c, layer, st);
  if (cudaMemsetAsync(v.head_done, 0, heads * sizeof(int), st) != cudaSuccess) return DMS_ERR_CUDA;
  if (launch_decode_attention(v, layer, q, o, c->has_maps ? &c->kmap : nullptr, c->has_maps ? &c->vmap : nullptr,
                              c->num_sms, st) != cudaSuccess)
    return DMS_ERR_CUDA;
  return DMS_OK;
}
