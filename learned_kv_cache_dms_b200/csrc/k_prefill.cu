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

constexpr int kScatterU = 4;  // 16-byte row chunks a thread loads before it stores any

// The replay runs in two launches over (chunk of kScanChunk tokens, (b, h)),
// so that a batch-1 prompt spreads over many SMs:
//   k_prefill_scan_bits   each chunk's evict, open and kept-list bits, their
//                         per-word prefixes within the chunk and the chunk's
//                         totals, into the layer's scan scratch (the first
//                         chunk also snapshots the ring and the counts);
//   k_prefill_scan_assign the chunks' totals summed in order, then every
//                         retained token of the chunk's slot (root walk over
//                         the head's bits) and kept-list entry; the last CTA
//                         grants pages in (b, h) order.
// A call at positions T0 .. T0 + T - 1 with T0 > 0 (a later chunk of a
// chunked prefill) continues from the layer's state:
//   open(t)  also holds when t - w < T0 and token t - w was kept;
//   root(t)  stops at the first r with r - w < T0: token r takes a fresh slot
//            (r open), or the slot of the marked token r - w (its ring entry);
//   fresh slots are numbered from the layer's count; kept-list entries from
//   the context's kept count (k_prefill_context).
constexpr int kScanChunk = 1024;  // tokens per CTA (32 words)
constexpr int kScanThreads = 256;

// Scan scratch of one (b, h): words of evict, open and kept-list bits and the
// open / kept-list prefixes of each word within its chunk, then per chunk the
// open and kept totals, the ring snapshot and the counts before the call.
struct ScanScratch {
  int nw, nc, w;
  unsigned *ev, *op, *kb;
  int *opre, *kpre, *ctot, *rs, *base;
  __device__ ScanScratch(const CacheView& c, int bh) {
    nw = (c.max_pos + 31) >> 5;
    nc = (c.max_pos + kScanChunk - 1) / kScanChunk;
    w = c.w;
    int* p = c.scan + static_cast<long>(bh) * c.scan_stride;
    ev = reinterpret_cast<unsigned*>(p);
    op = ev + nw;
    kb = op + nw;
    opre = reinterpret_cast<int*>(kb + nw);
    kpre = opre + nw;
    ctot = kpre + nw;  // [nc][2]
    rs = ctot + 2 * nc;
    base = rs + w;     // count0, kept0
  }
};

__global__ void __launch_bounds__(kScanThreads) k_prefill_scan_bits(CacheView c, int layer, int T0, int T,
                                                                    const float* alpha) {
  griddep_wait();
  griddep_launch_dependents();
  const int BH = c.B * c.Hkv;
  const int chunk = blockIdx.x, bh = blockIdx.y, b = bh / c.Hkv, h = bh % c.Hkv;
  const long lbh = static_cast<long>(layer) * BH + bh;
  const int hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
  const float* arow = alpha + (static_cast<long>(b) * c.Hkv + hs) * T;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int w = c.w, end = T0 + T;
  const int t0 = chunk * kScanChunk, t1 = min(T, t0 + kScanChunk);
  if (t0 >= T) return;
  ScanScratch sc(c, bh);
  const int* ring = c.ring + lbh * w;
  // decision shift +1: the mark of the call's first token is the previous
  // token's decision, carried from the previous call (0: the padding, keep)
  const bool carry_in = c.shift == 1 && T0 > 0 && c.carry[lbh] != 0;
  if (chunk == 0) {
    // what the assignment needs from before this call (it rewrites the ring)
    if (T0 > 0)
      for (int i = tid; i < w; i += kScanThreads) sc.rs[i] = ring[i];
    if (tid == 0) {
      sc.base[0] = T0 > 0 ? c.count[lbh] : 0;
      sc.base[1] = T0 > 0 ? c.kept_count[bh] : 0;
    }
  }
  // token t's eviction mark (0 <= t < T) is the decision of token t - shift:
  // +1 the previous token's (the carried one for t = 0), -1 the next token's
  // (none yet for the last)
  auto mark = [&](int t) {
    const int src = t - c.shift;
    return !c.disable && (src >= 0 && src < T ? arow[src] > 0.0f : (src < 0 && carry_in));
  };
  // evict, open and kept-list bits of the chunk's words (t the call's token
  // index, T0 + t its position); open(t) reads the mark of token t - w, in
  // this call or, before it, in the ring
  const int we = (t1 + 31) >> 5;
  for (int wi = (t0 >> 5) + wid; wi < we; wi += kScanThreads / 32) {
    const int t = wi * 32 + lane, e = T0 + t - w;
    bool ev = false, o = false, k = false;
    if (t < T) {
      ev = mark(t);
      const bool ev_e = e < 0 ? false : (e >= T0 ? mark(e - T0) : (ring[e % w] & static_cast<int>(RING_EVICT)) != 0);
      o = !ev_e;
      k = T0 + t < end - w && !ev;
    }
    const unsigned me = __ballot_sync(0xffffffffu, ev);
    const unsigned mo = __ballot_sync(0xffffffffu, o);
    const unsigned mk = __ballot_sync(0xffffffffu, k);
    if (lane == 0) {
      sc.ev[wi] = me;
      sc.op[wi] = mo;
      sc.kb[wi] = mk;
    }
  }
  __syncthreads();
  // prefixes within the chunk: warp 0, one word per lane (32 words per chunk)
  if (wid == 0) {
    const int wi = (t0 >> 5) + lane;
    const bool in = wi < we;
    const int po = in ? __popc(sc.op[wi]) : 0, pk = in ? __popc(sc.kb[wi]) : 0;
    int xo = po, xk = pk;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
      const int ao = __shfl_up_sync(0xffffffffu, xo, o2), ak = __shfl_up_sync(0xffffffffu, xk, o2);
      if (lane >= o2) {
        xo += ao;
        xk += ak;
      }
    }
    if (in) {
      sc.opre[wi] = xo - po;
      sc.kpre[wi] = xk - pk;
    }
    if (lane == 31) {
      sc.ctot[2 * chunk] = xo;
      sc.ctot[2 * chunk + 1] = xk;
    }
  }
}

__global__ void __launch_bounds__(kScanThreads) k_prefill_scan_assign(CacheView c, int layer, int T0, int T,
                                                                      const float* alpha) {
  extern __shared__ unsigned sm[];
  __shared__ int tmp[32];
  __shared__ int s_last;
  griddep_wait();
  griddep_launch_dependents();
  const int BH = c.B * c.Hkv;
  const int chunk = blockIdx.x, bh = blockIdx.y, b = bh / c.Hkv, h = bh % c.Hkv;
  const long lbh = static_cast<long>(layer) * BH + bh;
  const int hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
  const float* arow = alpha + (static_cast<long>(b) * c.Hkv + hs) * T;
  const int tid = threadIdx.x, bd = kScanThreads;
  const int w = c.w, end = T0 + T;
  const int t0 = chunk * kScanChunk, t1 = min(T, t0 + kScanChunk);
  const int nch = (T + kScanChunk - 1) / kScanChunk;
  ScanScratch sc(c, bh);
  // shared memory: evict, open bits and open prefixes of the words up to the
  // chunk's end (a root is at or before its token), the chunks' open and kept
  // bases, the ring snapshot
  const int nwu = (t1 + 31) >> 5;
  unsigned* ev = sm;
  unsigned* op = sm + nwu;
  int* opre = reinterpret_cast<int*>(sm + 2 * nwu);
  int* cbase = opre + nwu;  // [nch][2] exclusive bases, then the totals
  int* rs = cbase + 2 * nch + 2;
  if (t0 < T) {
    for (int i = tid; i < nwu; i += bd) {
      ev[i] = sc.ev[i];
      op[i] = sc.op[i];
      opre[i] = sc.opre[i];
    }
    if (T0 > 0)
      for (int i = tid; i < w; i += bd) rs[i] = sc.rs[i];
  }
  // the chunks' bases: an exclusive scan of their totals (every CTA alike)
  {
    int carry_o = 0, carry_k = 0;
    for (int i0 = 0; i0 < nch; i0 += bd) {
      const int i = i0 + tid;
      const int vo = i < nch ? sc.ctot[2 * i] : 0, vk = i < nch ? sc.ctot[2 * i + 1] : 0;
      int to, tk;
      const int xo = block_exclusive_scan(vo, tmp, &to);
      const int xk = block_exclusive_scan(vk, tmp, &tk);
      if (i < nch) {
        cbase[2 * i] = carry_o + xo;
        cbase[2 * i + 1] = carry_k + xk;
      }
      carry_o += to;
      carry_k += tk;
    }
    if (tid == 0) {
      cbase[2 * nch] = carry_o;
      cbase[2 * nch + 1] = carry_k;
    }
  }
  __syncthreads();
  const int count0 = sc.base[0], kept0 = sc.base[1];
  if (t0 < T) {
    // slots of the retained tokens; ring of the last w tokens; kept list
    auto evict_before = [&](int e) { return (rs[e % w] & static_cast<int>(RING_EVICT)) != 0; };
    int* slot_pos = c.slot_pos + lbh * c.cap;
    int* kept = c.kept + static_cast<long>(bh) * c.max_pos;
    int* kept_upto = c.kept_upto + static_cast<long>(bh) * (c.max_pos + 1);
    int* ring = c.ring + lbh * w;
    const int kbase = kept0 + cbase[2 * chunk + 1];
    for (int t = t0 + tid; t < t1; t += bd) {
      const int pos = T0 + t, wi = t >> 5;
      const bool evt = bit_at(ev, t);
      const unsigned below = (1u << (t & 31)) - 1u;
      const unsigned kbw = sc.kb[wi];
      const int kr = kbase + sc.kpre[wi] + __popc(kbw & below);
      kept_upto[pos] = kr;
      const bool retained = (pos >= end - w) || !evt;
      if (!retained) continue;
      int r = t;
      while (T0 + r - w >= T0 && bit_at(ev, r - w)) r -= w;
      const int e = T0 + r - w;
      int slot;
      if (e >= 0 && e < T0 && evict_before(e))
        slot = rs[e % w] & RING_SLOT_MASK;  // the marked token of the previous call leaves: its slot
      else
        slot = count0 + cbase[2 * (r / kScanChunk)] + opre[r >> 5] + __popc(op[r >> 5] & ((1u << (r & 31)) - 1u));
      slot_pos[slot] = pos;
      if (pos >= end - w) ring[pos % w] = slot | (evt ? static_cast<int>(RING_EVICT) : 0);
      if (pos < end - w) kept[kr] = pos;
    }
    if (chunk == nch - 1 && tid == 0) {
      const int tot_open = cbase[2 * nch], tot_keep = cbase[2 * nch + 1];
      kept_upto[end] = kept0 + tot_keep;
      c.count[lbh] = count0 + tot_open;
      c.kept_count[bh] = kept0 + tot_keep;
      if (c.shift == 1) c.carry[lbh] = (!c.disable && arow[T - 1] > 0.0f) ? 1 : 0;
      if (h == 0) c.pos[layer * c.B + b] = end;
    }
  }
  // the last CTA to arrive grants the extra pages of every head, in (b, h)
  // row-major order, from the ascending page counter
  __threadfence();
  __syncthreads();
  if (tid == 0)
    s_last = (atomicAdd(&c.ctrl[CTRL_DONE_SCAN], 1) == static_cast<int>(gridDim.x * gridDim.y) - 1);
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
  // slot plan of the first decode append (token end) of every head
  __syncthreads();
  for (int i = tid; i < BH; i += bd) {
    const long li = static_cast<long>(layer) * BH + i;
    *plan_at(c, li, end) = next_plan(c, li, end);
  }
}

size_t prefill_scan_smem(const CacheView& c, int T0, int T) {
  const size_t nwu = (static_cast<size_t>(T) + 31) / 32, nch = (static_cast<size_t>(T) + kScanChunk - 1) / kScanChunk;
  return (3 * nwu + 2 * nch + 2 + (T0 > 0 ? c.w : 0)) * 4;
}

int prefill_scan_stride(int max_pos, int w) {
  const int nw = (max_pos + 31) / 32, nc = (max_pos + kScanChunk - 1) / kScanChunk;
  return (5 * nw + 2 * nc + w + 2 + 7) / 8 * 8;
}

cudaError_t launch_prefill_scan(const CacheView& c, int layer, int T0, int T, const float* alpha, cudaStream_t s) {
  const dim3 grid((T + kScanChunk - 1) / kScanChunk, c.B * c.Hkv);
  // each launch a programmatic dependent of the one before it
  cudaError_t e = launch_dependent(k_prefill_scan_bits, grid, dim3(kScanThreads), 0, s, c, layer, T0, T, alpha);
  if (e != cudaSuccess) return e;
  const size_t smem = prefill_scan_smem(c, T0, T);
  e = cudaFuncSetAttribute(k_prefill_scan_assign, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_dependent(k_prefill_scan_assign, grid, dim3(kScanThreads), smem, s, c, layer, T0, T, alpha);
}

// ---------------------------------------------------------------------------
// Context of a prefill call into a layer that already holds T0 tokens (a later
// chunk of a chunked prefill), rebuilt from the cache before the call's
// compaction; one CTA per (b, h):
//  1. the position-sorted list of the kept tokens before T0: kept_upto[x] =
//     kept tokens at positions < x (x <= T0), kept[r] = the r-th kept
//     position, and their K/V rows in the kept copy in that order.  A token
//     held at position j < T0 - w is kept (a marked one would have been
//     overwritten); a younger one is kept or marked as its ring entry says;
//  2. the K/V rows of the last w positions T0 - w .. T0 - 1 in position order
//     (window copy): the band keys the call's first queries see before its
//     own.
// The kept list and kept copy are scratch shared by the layers, so every call
// rebuilds them for its own layer.  Rows are bf16: FP8 pages are decoded with
// their page scale and rounded.
// ---------------------------------------------------------------------------
template <bool FP8>
__device__ __forceinline__ uint4 page_row_chunk(const CacheView& c, const void* pool, const float* scales, int id,
                                                int row, int ch) {
  if (!FP8) {
    return reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(pool) +
                                          (static_cast<long>(id) * c.P + row) * c.D)[ch];
  } else {
    const uint2 q = reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(pool) +
                                                   (static_cast<long>(id) * c.P + row) * c.D)[ch];
    const float sc = scales[id];
    float f[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = fp8_decode(static_cast<uint8_t>(((e < 4 ? q.x : q.y) >> (8 * (e & 3))) & 0xFF)) * sc;
    return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
  }
}

template <bool FP8>
__global__ void __launch_bounds__(1024) k_prefill_context(CacheView c, int layer, int T0, int T, const float* alpha) {
  __shared__ int tmp[32];
  const int bh = blockIdx.x, tid = threadIdx.x, bd = blockDim.x, w = c.w;
  const long lbh = static_cast<long>(layer) * c.B * c.Hkv + bh;
  const int count0 = c.count[lbh];
  int* kept_upto = c.kept_upto + static_cast<long>(bh) * (c.max_pos + 1);
  int* kept = c.kept + static_cast<long>(bh) * c.max_pos;
  const int* slot_pos = c.slot_pos + lbh * c.cap;
  int* ring = c.ring + lbh * w;
  const int* pt = c.page_table + lbh * c.maxp;
  // decision shift -1: the call's first decision marks the layer's last token
  if (c.shift == -1 && tid == 0) {
    const int b = bh / c.Hkv, hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : bh % c.Hkv;
    if (!c.disable && alpha[(static_cast<long>(b) * c.Hkv + hs) * T] > 0.0f)
      ring[(T0 - 1) % w] |= static_cast<int>(RING_EVICT);
  }
  __syncthreads();
  auto is_kept = [&](int j) { return j < T0 - w || (ring[j % w] & static_cast<int>(RING_EVICT)) == 0; };
  // 1. flags at the kept positions, then an exclusive scan in place
  for (int x = tid; x <= T0; x += bd) kept_upto[x] = 0;
  __syncthreads();
  for (int s = tid; s < count0; s += bd) {
    const int j = slot_pos[s];
    if (is_kept(j)) kept_upto[j] = 1;
  }
  __syncthreads();
  const int n = T0 + 1, per = (n + bd - 1) / bd;
  const int x0 = min(n, tid * per), x1 = min(n, x0 + per);
  int sum = 0;
  for (int x = x0; x < x1; ++x) sum += kept_upto[x];
  int total;
  int base = block_exclusive_scan(sum, tmp, &total);
  for (int x = x0; x < x1; ++x) {
    const int f = kept_upto[x];
    kept_upto[x] = base;
    base += f;
  }
  __syncthreads();
  if (tid == 0) c.kept_count[bh] = total;
  // kept list and kept copy (16-byte chunks of bf16 rows)
  const int cpr = c.D / 8;
  __nv_bfloat16* kk = static_cast<__nv_bfloat16*>(c.kept_k) + static_cast<long>(bh) * c.max_pos * c.D;
  __nv_bfloat16* kv = static_cast<__nv_bfloat16*>(c.kept_v) + static_cast<long>(bh) * c.max_pos * c.D;
  for (int idx = tid; idx < count0 * cpr; idx += bd) {
    const int s = idx / cpr, ch = idx % cpr;
    const int j = slot_pos[s];
    if (!is_kept(j)) continue;
    const int r = kept_upto[j];
    if (ch == 0) kept[r] = j;
    const int id = pt[s / c.P];
    if (id < 0) continue;  // no page (pool exhausted): the status word says so
    reinterpret_cast<uint4*>(kk + static_cast<long>(r) * c.D)[ch] =
        page_row_chunk<FP8>(c, c.k_pool, c.k_scale, id, s % c.P, ch);
    reinterpret_cast<uint4*>(kv + static_cast<long>(r) * c.D)[ch] =
        page_row_chunk<FP8>(c, c.v_pool, c.v_scale, id, s % c.P, ch);
  }
  // 2. window copy: position T0 - w + i at row i
  __nv_bfloat16* wk = static_cast<__nv_bfloat16*>(c.win_k) + static_cast<long>(bh) * w * c.D;
  __nv_bfloat16* wv = static_cast<__nv_bfloat16*>(c.win_v) + static_cast<long>(bh) * w * c.D;
  for (int idx = tid; idx < w * cpr; idx += bd) {
    const int i = idx / cpr, ch = idx % cpr, j = T0 - w + i;
    if (j < 0) continue;
    const int s = ring[j % w] & RING_SLOT_MASK;
    const int id = pt[s / c.P];
    if (id < 0) continue;
    reinterpret_cast<uint4*>(wk + static_cast<long>(i) * c.D)[ch] =
        page_row_chunk<FP8>(c, c.k_pool, c.k_scale, id, s % c.P, ch);
    reinterpret_cast<uint4*>(wv + static_cast<long>(i) * c.D)[ch] =
        page_row_chunk<FP8>(c, c.v_pool, c.v_scale, id, s % c.P, ch);
  }
}

cudaError_t launch_prefill_context(const CacheView& c, int layer, int T0, int T, const float* alpha, cudaStream_t s) {
  if (c.kv_dtype == DMS_FP8_E4M3)
    k_prefill_context<true><<<c.B * c.Hkv, 1024, 0, s>>>(c, layer, T0, T, alpha);
  else
    k_prefill_context<false><<<c.B * c.Hkv, 1024, 0, s>>>(c, layer, T0, T, alpha);
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
// With T0 > 0 (a later chunk) only slots holding this call's tokens (positions
// >= T0) are written; the others keep their rows.
template <typename TA>
__global__ void __launch_bounds__(256) k_prefill_scatter(CacheView c, int layer, int T0, int T, int rg, const TA* k,
                                                         const TA* v) {
  griddep_wait();
  griddep_launch_dependents();
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
      tt[u] = idx < n ? slot_pos[idx / cpr] - T0 : -1;  // the call's token index (< 0: an older row)
    }
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      if (tt[u] < 0) continue;
      const int ch = (base + u * blockDim.x) % cpr;
      const long src = ((static_cast<long>(b) * T + tt[u]) * c.Hkv + h) * c.D;
      kq[u] = reinterpret_cast<const uint4*>(k + src)[ch];
      vq[u] = reinterpret_cast<const uint4*>(v + src)[ch];
      kr[u] = kept_copy && tt[u] < T - c.w ? kept_upto[T0 + tt[u]] : -1;
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

// With T0 > 0 (a later chunk) a page may already hold rows of earlier calls
// ("old" rows, positions < T0): its scale becomes max(old scale, amax of the
// new rows / 448) and, when it grows, the old rows are first re-encoded from
// their decoded values (code' = RNE(fl32(fl32(dec(code) * s_old) / s_new))),
// the decode append's rule applied once for the call; pages without new rows
// are left as they are.
__global__ void __launch_bounds__(256) k_prefill_scatter_fp8(CacheView c, int layer, int T0, int T,
                                                            const __nv_bfloat16* k, const __nv_bfloat16* v) {
  __shared__ float red[32];
  griddep_wait();
  griddep_launch_dependents();
  const int p = blockIdx.x, bh = blockIdx.y;
  const int b = bh / c.Hkv, h = bh % c.Hkv;
  const long lbh = static_cast<long>(layer) * c.B * c.Hkv + bh;
  const int cnt = c.count[lbh];
  if (p * c.P >= cnt) return;
  const int id = c.page_table[lbh * c.maxp + p];
  if (id < 0) return;
  const int rows = min(c.P, cnt - p * c.P);
  const int* slot_pos = c.slot_pos + lbh * c.cap + static_cast<long>(p) * c.P;
  // which rows this call wrote (new) and which it did not (old)
  bool any_new = false, any_old = false;
  for (int r = threadIdx.x; r < rows; r += blockDim.x) (slot_pos[r] >= T0 ? any_new : any_old) = true;
  any_new = __syncthreads_or(any_new);
  any_old = __syncthreads_or(any_old);
  if (!any_new) return;
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
      tt[u] = idx < n ? slot_pos[idx / cpr] - T0 : -1;  // the call's token index (< 0: an old row)
    }
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      if (tt[u] < 0) continue;
      const int ch = (base + u * blockDim.x) % cpr;
      const long src = ((static_cast<long>(b) * T + tt[u]) * c.Hkv + h) * c.D;
      kq[u] = reinterpret_cast<const uint4*>(k + src)[ch];
      vq[u] = reinterpret_cast<const uint4*>(v + src)[ch];
      kr[u] = kept_copy && tt[u] < T - c.w ? kept_upto[T0 + tt[u]] : -1;
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
  const float sk_old = any_old ? c.k_scale[id] : 0.f, sv_old = any_old ? c.v_scale[id] : 0.f;
  const float sk = fmaxf(sk_old, __fdiv_rn(ak, 448.0f)), sv = fmaxf(sv_old, __fdiv_rn(av, 448.0f));
  uint8_t* kd = static_cast<uint8_t*>(c.k_pool) + static_cast<long>(id) * c.P * c.D;
  uint8_t* vd = static_cast<uint8_t*>(c.v_pool) + static_cast<long>(id) * c.P * c.D;
  // old rows at a grown scale: re-encoded from their decoded values
  const bool grow_k = any_old && sk > sk_old, grow_v = any_old && sv > sv_old;
  if (grow_k || grow_v) {
    for (int idx = threadIdx.x; idx < rows * c.D; idx += blockDim.x) {
      if (slot_pos[idx / c.D] >= T0) continue;
      if (grow_k) kd[idx] = fp8_encode(__fdiv_rn(__fmul_rn(fp8_decode(kd[idx]), sk_old), sk));
      if (grow_v) vd[idx] = fp8_encode(__fdiv_rn(__fmul_rn(fp8_decode(vd[idx]), sv_old), sv));
    }
  }
  if (threadIdx.x == 0) {
    c.k_scale[id] = sk;
    c.v_scale[id] = sv;
  }
  for (int base = threadIdx.x; base < n; base += kScatterU * blockDim.x) {
    int tt[kScatterU];
    uint4 kq[kScatterU], vq[kScatterU];
#pragma unroll
    for (int u = 0; u < kScatterU; ++u) {
      const int idx = base + u * blockDim.x;
      tt[u] = idx < n ? slot_pos[idx / cpr] - T0 : -1;
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

cudaError_t launch_prefill_scatter(const CacheView& c, int layer, int T0, int T, const void* k, const void* v,
                                   cudaStream_t s) {
  // pages that can hold the call's tokens: every page up to the layer's
  // count (slots reused in place may sit in any earlier page)
  const int pages = min(c.maxp, (T0 + T + c.P - 1) / c.P);
  if (c.kv_dtype == DMS_FP8_E4M3) {
    return launch_dependent(k_prefill_scatter_fp8, dim3(pages, c.B * c.Hkv), dim3(256), 0, s, c, layer, T0, T,
                            static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v));
  }
  // rows per CTA: one batch of kScatterU chunks per thread
  const int cpr = c.D * (c.kv_dtype == DMS_BF16 ? 2 : 4) / 16;
  const int rg = max(1, min(c.P, kScatterU * 256 / cpr));
  dim3 grid(pages * ((c.P + rg - 1) / rg), c.B * c.Hkv);
  if (c.kv_dtype == DMS_BF16)
    return launch_dependent(k_prefill_scatter<__nv_bfloat16>, grid, dim3(256), 0, s, c, layer, T0, T, rg,
                            static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v));
  return launch_dependent(k_prefill_scatter<float>, grid, dim3(256), 0, s, c, layer, T0, T, rg,
                          static_cast<const float*>(k), static_cast<const float*>(v));
}

}  // namespace dms
