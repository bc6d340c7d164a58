// Prefill compaction: the append rule of the paged DMS cache replayed for all T
// prompt tokens at once, then the survivors streamed into their pages.
//
// Sequentially ([DMS-Qwen3], inference mode with the paged cache), token t
// takes the slot of token t - w when that token was marked for eviction, and a
// fresh slot otherwise.  In parallel form:
//   open(t)    = t < w  or  evict(t - w) == 0      (t takes a fresh slot)
//   newslot(t) = number of open tokens before t     (exclusive scan)
//   root(t)    = t if open(t) else root(t - w)      (walk back in steps of w)
//   slot(t)    = newslot(root(t))
// The final occupants are the last w tokens plus every earlier kept token, so
// only those are written; count = number of open tokens.
#include "decode_common.cuh"

namespace dms {

__device__ __forceinline__ bool bit_at(const unsigned* bits, int t) { return (bits[t >> 5] >> (t & 31)) & 1u; }

constexpr int kScanU = 16;    // decision-logit words a warp loads before its ballots
constexpr int kScatterU = 4;  // 16-byte row chunks a thread loads before it stores any

// One CTA per (b, h).  Shared memory: five arrays of ceil(T/32) words.
__global__ void __launch_bounds__(1024) k_prefill_scan(CacheView c, int layer, int T, const float* alpha) {
  extern __shared__ unsigned sm[];
  const int nw = (T + 31) >> 5;
  unsigned* ev = sm;                                       // evict bits
  unsigned* op = sm + nw;                                  // open bits
  unsigned* kb = sm + 2 * nw;                              // kept-list bits: kept and t < T - w
  int* opre = reinterpret_cast<int*>(sm + 3 * nw);         // exclusive prefix of open bits per word
  int* kpre = reinterpret_cast<int*>(sm + 4 * nw);         // exclusive prefix of kept-list bits per word
  __shared__ int tmp[32];
  __shared__ int s_last;

  const int BH = c.B * c.Hkv;
  const int bh = blockIdx.x, b = bh / c.Hkv, h = bh % c.Hkv;
  const long lbh = static_cast<long>(layer) * BH + bh;
  const int hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
  const float* arow = alpha + (static_cast<long>(b) * c.Hkv + hs) * T;
  const int tid = threadIdx.x, lane = tid & 31, bd = blockDim.x;
  const int w = c.w;

  // 1. evict bits (coalesced read, one ballot per 32 tokens).  Warp wid owns
  //    words wid, wid + nwarp, ...; it issues the loads of kScanU words before
  //    the first ballot so that they are in flight together.
  const int wid = tid >> 5, nwarp = bd >> 5;
  for (int w0 = wid; w0 < nw; w0 += nwarp * kScanU) {
    bool e[kScanU];
#pragma unroll
    for (int u = 0; u < kScanU; ++u) {
      const int t = (w0 + u * nwarp) * 32 + lane;
      e[u] = t < T && arow[t] > 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kScanU; ++u) {
      const unsigned m = __ballot_sync(0xffffffffu, e[u] && !c.disable);
      if (lane == 0 && w0 + u * nwarp < nw) ev[w0 + u * nwarp] = m;
    }
  }
  __syncthreads();
  // 2. open bits and kept-list bits
  for (int t0 = (tid & ~31); t0 < nw * 32; t0 += bd) {
    const int t = t0 + lane;
    const bool o = t < T && (t < w || !bit_at(ev, t - w));
    const bool k = t < T - w && !bit_at(ev, t);
    const unsigned mo = __ballot_sync(0xffffffffu, o);
    const unsigned mk = __ballot_sync(0xffffffffu, k);
    if (lane == 0) {
      op[t0 >> 5] = mo;
      kb[t0 >> 5] = mk;
    }
  }
  __syncthreads();
  // 3. exclusive scans over words: each thread owns a contiguous run
  const int per = (nw + bd - 1) / bd;
  const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
  int so = 0, sk = 0;
  for (int i = w0; i < w1; ++i) {
    so += __popc(op[i]);
    sk += __popc(kb[i]);
  }
  int tot_open, tot_keep;
  int base_o = block_exclusive_scan(so, tmp, &tot_open);
  int base_k = block_exclusive_scan(sk, tmp, &tot_keep);
  for (int i = w0; i < w1; ++i) {
    opre[i] = base_o;
    kpre[i] = base_k;
    base_o += __popc(op[i]);
    base_k += __popc(kb[i]);
  }
  __syncthreads();
  // 4. slots of the retained tokens; ring of the last w tokens; kept list
  int* slot_pos = c.slot_pos + lbh * c.cap;
  int* ring = c.ring + lbh * w;
  int* kept = c.kept + static_cast<long>(bh) * c.max_pos;
  int* kept_upto = c.kept_upto + static_cast<long>(bh) * (c.max_pos + 1);
  for (int t = tid; t < T; t += bd) {
    const bool evt = bit_at(ev, t);
    const unsigned below = (1u << (t & 31)) - 1u;
    kept_upto[t] = kpre[t >> 5] + __popc(kb[t >> 5] & below);
    const bool retained = (t >= T - w) || !evt;
    if (!retained) continue;
    int r = t;
    while (r >= w && bit_at(ev, r - w)) r -= w;
    const int slot = opre[r >> 5] + __popc(op[r >> 5] & ((1u << (r & 31)) - 1u));
    slot_pos[slot] = t;
    if (t >= T - w) ring[t % w] = slot | (evt ? static_cast<int>(RING_EVICT) : 0);
    if (t < T - w) kept[kpre[t >> 5] + __popc(kb[t >> 5] & below)] = t;
  }
  if (tid == 0) {
    kept_upto[T] = tot_keep;
    c.count[lbh] = tot_open;
    c.kept_count[bh] = tot_keep;
    if (h == 0) c.pos[layer * c.B + b] = T;
  }
  // 5. the last CTA to arrive grants the extra pages of every head, in (b, h)
  //    row-major order, from the ascending page counter.
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&c.ctrl[CTRL_DONE_SCAN], 1) == static_cast<int>(gridDim.x) - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  int next = __ldcg(&c.ctrl[CTRL_NEXT_PAGE]);
  for (int i0 = 0; i0 < BH; i0 += bd) {
    const int i = i0 + tid;
    int need = 0, have = 0;
    const long li = static_cast<long>(layer) * BH + i;
    if (i < BH) {
      const int cnt = __ldcg(&c.count[li]);
      have = c.npages[li];
      need = max(0, (cnt + c.P - 1) / c.P - have);
    }
    int tot;
    const int off = block_exclusive_scan(need, tmp, &tot);
    int granted = 0;
    for (int j = 0; j < need; ++j) {
      const int id = next + off + j;
      if (id < c.pool_pages && have + j < c.maxp) {
        c.page_table[li * c.maxp + have + j] = id;
        ++granted;
      } else {
        set_status(c.ctrl, DMS_ST_POOL_EXHAUSTED);
      }
    }
    if (i < BH) c.npages[li] = have + granted;
    next += tot;
  }
  if (tid == 0) {
    c.ctrl[CTRL_NEXT_PAGE] = min(next, c.pool_pages);
    c.ctrl[CTRL_DONE_SCAN] = 0;
  }
  // slot plan of the first decode append (token T) of every head
  __syncthreads();
  for (int i = tid; i < BH; i += bd) {
    const long li = static_cast<long>(layer) * BH + i;
    *plan_at(c, li, T) = next_plan(c, li, T);
  }
}

cudaError_t launch_prefill_scan(const CacheView& c, int layer, int T, const float* alpha, cudaStream_t s) {
  const int nw = (T + 31) / 32;
  const size_t smem = static_cast<size_t>(nw) * 5 * 4;
  cudaError_t e = cudaFuncSetAttribute(k_prefill_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  k_prefill_scan<<<c.B * c.Hkv, 1024, smem, s>>>(c, layer, T, alpha);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Scatter of the survivors into their pages.  Slot s of a page holds token
// slot_pos[s]; rows are copied as 16-byte chunks.  FP8 pages: scale = max |x| /
// 448 over the page's rows (K and V separately), code = RNE-satfinite(x /
// scale); eviction is applied before quantisation ([FastDMS], quality section).
//
// Every thread gathers up to kScatterU chunks per batch: the slot positions,
// then the K/V chunks (and the kept-list ranks), all loads issued before the
// first store, so a batch costs two dependent DRAM round trips.
// ---------------------------------------------------------------------------

// bf16 / fp32 pages: one CTA per (group of rg rows of a page, (b, h)), with
// rg * 16-byte chunks per row <= kScatterU * blockDim.x (one batch per thread).
template <typename TA>
__global__ void __launch_bounds__(256) k_prefill_scatter(CacheView c, int layer, int T, int rg, const TA* k,
                                                         const TA* v) {
  const int gpp = (c.P + rg - 1) / rg;
  const int p = blockIdx.x / gpp, r0 = (blockIdx.x % gpp) * rg, bh = blockIdx.y;
  const int b = bh / c.Hkv, h = bh % c.Hkv;
  const long lbh = static_cast<long>(layer) * c.B * c.Hkv + bh;
  const int cnt = c.count[lbh];
  const int s0 = p * c.P + r0;  // first slot of this CTA
  if (s0 >= cnt) return;
  const int id = c.page_table[lbh * c.maxp + p];
  if (id < 0) return;
  const int rows = min(rg, min(c.P - r0, cnt - s0));
  const int* slot_pos = c.slot_pos + lbh * c.cap + s0;
  constexpr int V = 16 / sizeof(TA);
  const int cpr = c.D / V;  // 16-byte chunks per row
  TA* kp = static_cast<TA*>(c.k_pool) + (static_cast<long>(id) * c.P + r0) * c.D;
  TA* vp = static_cast<TA*>(c.v_pool) + (static_cast<long>(id) * c.P + r0) * c.D;
  const int* kept_upto = c.kept_upto + static_cast<long>(bh) * (c.max_pos + 1);
  // a kept token before the last window also goes into the position-sorted
  // kept copy read by the tcgen05 prefill attention
  const bool kept_copy = sizeof(TA) == 2 && c.kept_k != nullptr;
  const int n = rows * cpr;
  for (int base = threadIdx.x; base < n; base += kScatterU * blockDim.x) {
    int tt[kScatterU], kr[kScatterU];
    uint4 kq[kScatterU], vq[kScatterU];
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      const int idx = base + u * blockDim.x;
      tt[u] = idx < n ? slot_pos[idx / cpr] : -1;
    }
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      if (tt[u] < 0) continue;
      const int ch = (base + u * blockDim.x) % cpr;
      const long src = ((static_cast<long>(b) * T + tt[u]) * c.Hkv + h) * c.D;
      kq[u] = reinterpret_cast<const uint4*>(k + src)[ch];
      vq[u] = reinterpret_cast<const uint4*>(v + src)[ch];
      kr[u] = kept_copy && tt[u] < T - c.w ? kept_upto[tt[u]] : -1;
    }
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      if (tt[u] < 0) continue;
      const int idx = base + u * blockDim.x, r = idx / cpr, ch = idx % cpr;
      reinterpret_cast<uint4*>(kp + static_cast<long>(r) * c.D)[ch] = kq[u];
      reinterpret_cast<uint4*>(vp + static_cast<long>(r) * c.D)[ch] = vq[u];
      if (kr[u] >= 0) {
        const long dst = (static_cast<long>(bh) * c.max_pos + kr[u]) * c.D;
        reinterpret_cast<uint4*>(static_cast<TA*>(c.kept_k) + dst)[ch] = kq[u];
        reinterpret_cast<uint4*>(static_cast<TA*>(c.kept_v) + dst)[ch] = vq[u];
      }
    }
  }
}

__device__ __forceinline__ float block_max(float x, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) red[wid] = x;
  __syncthreads();
  float m = 0.f;
  for (int i = 0; i < (blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  return m;
}

// FP8 pages: one CTA per (page, (b, h)); the scale needs the whole page.  Pass 1
// takes max |x| of K and V and writes the kept copy; pass 2 re-reads the rows
// (now in L2) and writes the codes.
__device__ __forceinline__ uint2 encode8(const uint4 x, float scale) {
  float f[8];
  unpack16(x, f, static_cast<const __nv_bfloat16*>(nullptr));
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t q = scale > 0.f ? fp8_encode(__fdiv_rn(f[e], scale)) : 0u;
    if (e < 4)
      lo |= q << (8 * e);
    else
      hi |= q << (8 * (e - 4));
  }
  return make_uint2(lo, hi);
}

__device__ __forceinline__ float amax8(const uint4 x, float m) {
  float f[8];
  unpack16(x, f, static_cast<const __nv_bfloat16*>(nullptr));
#pragma unroll
  for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
  return m;
}

__global__ void __launch_bounds__(256) k_prefill_scatter_fp8(CacheView c, int layer, int T, const __nv_bfloat16* k,
                                                            const __nv_bfloat16* v) {
  __shared__ float red[32];
  const int p = blockIdx.x, bh = blockIdx.y;
  const int b = bh / c.Hkv, h = bh % c.Hkv;
  const long lbh = static_cast<long>(layer) * c.B * c.Hkv + bh;
  const int cnt = c.count[lbh];
  if (p * c.P >= cnt) return;
  const int id = c.page_table[lbh * c.maxp + p];
  if (id < 0) return;
  const int rows = min(c.P, cnt - p * c.P);
  const int* slot_pos = c.slot_pos + lbh * c.cap + static_cast<long>(p) * c.P;
  const int cpr = c.D / 8;  // 8 bf16 per 16-byte input chunk
  const int n = rows * cpr;
  const int* kept_upto = c.kept_upto + static_cast<long>(bh) * (c.max_pos + 1);
  const bool kept_copy = c.kept_k != nullptr;
  float ak = 0.f, av = 0.f;
  for (int base = threadIdx.x; base < n; base += kScatterU * blockDim.x) {
    int tt[kScatterU], kr[kScatterU];
    uint4 kq[kScatterU], vq[kScatterU];
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      const int idx = base + u * blockDim.x;
      tt[u] = idx < n ? slot_pos[idx / cpr] : -1;
    }
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      if (tt[u] < 0) continue;
      const int ch = (base + u * blockDim.x) % cpr;
      const long src = ((static_cast<long>(b) * T + tt[u]) * c.Hkv + h) * c.D;
      kq[u] = reinterpret_cast<const uint4*>(k + src)[ch];
      vq[u] = reinterpret_cast<const uint4*>(v + src)[ch];
      kr[u] = kept_copy && tt[u] < T - c.w ? kept_upto[tt[u]] : -1;
    }
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      if (tt[u] < 0) continue;
      ak = amax8(kq[u], ak);
      av = amax8(vq[u], av);
      if (kr[u] >= 0) {
        // kept tokens before the last window: into the position-sorted kept copy
        const int ch = (base + u * blockDim.x) % cpr;
        const long dst = (static_cast<long>(bh) * c.max_pos + kr[u]) * c.D;
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.kept_k) + dst)[ch] = kq[u];
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.kept_v) + dst)[ch] = vq[u];
      }
    }
  }
  ak = block_max(ak, red);
  av = block_max(av, red);
  const float sk = __fdiv_rn(ak, 448.0f), sv = __fdiv_rn(av, 448.0f);
  if (threadIdx.x == 0) {
    c.k_scale[id] = sk;
    c.v_scale[id] = sv;
  }
  uint8_t* kd = static_cast<uint8_t*>(c.k_pool) + static_cast<long>(id) * c.P * c.D;
  uint8_t* vd = static_cast<uint8_t*>(c.v_pool) + static_cast<long>(id) * c.P * c.D;
  for (int base = threadIdx.x; base < n; base += kScatterU * blockDim.x) {
    int tt[kScatterU];
    uint4 kq[kScatterU], vq[kScatterU];
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      const int idx = base + u * blockDim.x;
      tt[u] = idx < n ? slot_pos[idx / cpr] : -1;
    }
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      if (tt[u] < 0) continue;
      const int ch = (base + u * blockDim.x) % cpr;
      const long src = ((static_cast<long>(b) * T + tt[u]) * c.Hkv + h) * c.D;
      kq[u] = reinterpret_cast<const uint4*>(k + src)[ch];
      vq[u] = reinterpret_cast<const uint4*>(v + src)[ch];
    }
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      if (tt[u] < 0) continue;
      const int idx = base + u * blockDim.x, r = idx / cpr, ch = idx % cpr;
      reinterpret_cast<uint2*>(kd + static_cast<long>(r) * c.D)[ch] = encode8(kq[u], sk);
      reinterpret_cast<uint2*>(vd + static_cast<long>(r) * c.D)[ch] = encode8(vq[u], sv);
    }
  }
}

cudaError_t launch_prefill_scatter(const CacheView& c, int layer, int T, const void* k, const void* v,
                                   cudaStream_t s) {
  const int pages = min(c.maxp, (T + c.P - 1) / c.P);
  if (c.kv_dtype == DMS_FP8_E4M3) {
    k_prefill_scatter_fp8<<<dim3(pages, c.B * c.Hkv), 256, 0, s>>>(c, layer, T, static_cast<const __nv_bfloat16*>(k),
                                                                   static_cast<const __nv_bfloat16*>(v));
    return cudaGetLastError();
  }
  // rows per CTA: one batch of kScatterU chunks per thread
  const int cpr = c.D * (c.kv_dtype == DMS_BF16 ? 2 : 4) / 16;
  const int rg = max(1, min(c.P, kScatterU * 256 / cpr));
  dim3 grid(pages * ((c.P + rg - 1) / rg), c.B * c.Hkv);
  if (c.kv_dtype == DMS_BF16)
    k_prefill_scatter<__nv_bfloat16><<<grid, 256, 0, s>>>(c, layer, T, rg, static_cast<const __nv_bfloat16*>(k),
                                                          static_cast<const __nv_bfloat16*>(v));
  else
    k_prefill_scatter<float><<<grid, 256, 0, s>>>(c, layer, T, rg, static_cast<const float*>(k),
                                                  static_cast<const float*>(v));
  return cudaGetLastError();
}

}  // namespace dms
