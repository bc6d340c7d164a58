// Cache initialisation, decision logits and the neuron / rotary pre-pass.
#include "dms_internal.cuh"

namespace dms {

// ---------------------------------------------------------------------------
// Initialise (or reset) a cache: positions and counts to zero, preallocated
// pages granted row-major over (layer, batch, kv-head, page), page scales to
// zero, control words cleared, the page counter at the first free page.
// ---------------------------------------------------------------------------
__global__ void k_init(CacheView c) {
  const long nbh = static_cast<long>(c.L) * c.B * c.Hkv;
  const long npt = nbh * c.maxp;
  const long n = max(max(npt, static_cast<long>(c.pool_pages)), static_cast<long>(CTRL_WORDS));
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    if (i < npt) {
      const long lbh = i / c.maxp;
      const int p = static_cast<int>(i % c.maxp);
      c.page_table[i] = p < c.pre_pages ? static_cast<int>(lbh * c.pre_pages + p) : -1;
    }
    if (i < nbh) {
      c.npages[i] = c.pre_pages;
      c.count[i] = 0;
      c.carry[i] = 0;
      c.plan[i] = make_int4(0, 0, 0, 0);
      c.plan[nbh + i] = make_int4(0, 0, 0, 0);
    }
    if (i < static_cast<long>(c.B) * c.Hkv) c.head_done[i] = 0;
    if (i < static_cast<long>(c.L) * c.B) c.pos[i] = 0;
    if (i < c.pool_pages) {
      c.k_scale[i] = 0.0f;
      c.v_scale[i] = 0.0f;
    }
    if (i < CTRL_WORDS) c.ctrl[i] = (i == CTRL_NEXT_PAGE) ? static_cast<int>(nbh * c.pre_pages) : 0;
  }
}

cudaError_t launch_init(const CacheView& c, bool full, cudaStream_t s) {
  if (full) {
    // Zero the page pools once: rows past a head's count are read (and masked)
    // by the attention tiles, so they must hold finite values.
    const size_t eb = c.kv_dtype == DMS_F32 ? 4 : c.kv_dtype == DMS_BF16 ? 2 : 1;
    const size_t pool_bytes = static_cast<size_t>(c.pool_pages) * c.P * c.D * eb;
    cudaError_t e = cudaMemsetAsync(c.k_pool, 0, pool_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(c.v_pool, 0, pool_bytes, s);
    // the kept copies too: tiles read (and mask) rows past the kept count
    const size_t kept_bytes = static_cast<size_t>(c.B) * c.Hkv * c.max_pos * c.D * 2;
    if (e == cudaSuccess && c.kept_k) e = cudaMemsetAsync(c.kept_k, 0, kept_bytes, s);
    if (e == cudaSuccess && c.kept_v) e = cudaMemsetAsync(c.kept_v, 0, kept_bytes, s);
    // and the window copies (rows of positions before 0 are read and masked)
    const size_t win_bytes = static_cast<size_t>(c.B) * c.Hkv * c.w * c.D * 2;
    if (e == cudaSuccess && c.win_k) e = cudaMemsetAsync(c.win_k, 0, win_bytes, s);
    if (e == cudaSuccess && c.win_v) e = cudaMemsetAsync(c.win_v, 0, win_bytes, s);
    if (e != cudaSuccess) return e;
  }
  const long nbh = static_cast<long>(c.L) * c.B * c.Hkv;
  const long n = max(max(nbh * c.maxp, static_cast<long>(c.pool_pages)), static_cast<long>(CTRL_WORDS));
  const int grid = static_cast<int>(min((n + 255) / 256, 4096L));
  k_init<<<grid, 256, 0, s>>>(c);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Decision logits from the adapter: alpha = (W_h . RMSNorm_gamma(x) + bias_h)
// * scale - offset.  RMSNorm's gamma is folded into W in shared memory, and the
// 1/rms factor is applied after the dot product:
//   W_h . (x * inv * gamma) = inv * ((W_h * gamma) . x).
// Each warp handles kTok tokens at once so each W element read from shared
// memory serves kTok tokens, and requests the hidden rows kUnroll 16-byte
// vectors ahead per lane so enough bytes are in flight to stream them at HBM
// speed.  The folded table is filled with 16-byte loads.  Supports Hkv <= 8.
// ---------------------------------------------------------------------------
constexpr int kTok = 4;
constexpr int kUnroll = 4;

template <typename TA>
__global__ void __launch_bounds__(256) k_decide_proj(CacheView c, int T, DecideArgs a, float* alpha) {
  extern __shared__ float wg[];  // [Hkv][hidden]
  const int H = c.Hkv, hid = c.hidden;
  const TA* W = static_cast<const TA*>(a.W);
  const TA* gamma = static_cast<const TA*>(a.gamma);
  const TA* hs = static_cast<const TA*>(a.hidden);
  const TA* bias = static_cast<const TA*>(a.bias);
  constexpr int V = 16 / sizeof(TA);
  const int nvec = hid / V;
#pragma unroll 8
  for (int i = threadIdx.x; i < H * nvec; i += blockDim.x) {
    float wv[V], gv[V];
    unpack16(reinterpret_cast<const uint4*>(W)[i], wv, static_cast<const TA*>(nullptr));
    unpack16(gamma16<TA>(gamma, i % nvec), gv, static_cast<const TA*>(nullptr));
#pragma unroll
    for (int e = 0; e < V; ++e) wg[i * V + e] = wv[e] * gv[e];
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long gw = static_cast<long>(blockIdx.x) * warps + (threadIdx.x >> 5);
  const long nwarps = static_cast<long>(gridDim.x) * warps;
  const long ntok = static_cast<long>(c.B) * T;
  const bool layer_mode = c.alpha_per == DMS_ALPHA_PER_LAYER;

  for (long tok0 = gw * kTok; tok0 < ntok; tok0 += nwarps * kTok) {
    float ss[kTok];
    float dot[kTok][8];
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
      ss[u] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) dot[u][j] = 0.f;
    }
    for (int vb = 0; vb < nvec; vb += 32 * kUnroll) {
      // every load of the block first, then the arithmetic
      uint4 raw[kUnroll][kTok];
#pragma unroll
      for (int k = 0; k < kUnroll; ++k) {
        const int vi = vb + k * 32 + lane;
#pragma unroll
        for (int u = 0; u < kTok; ++u) {
          const long tok = tok0 + u;
          raw[k][u] = (vi < nvec && tok < ntok) ? reinterpret_cast<const uint4*>(hs + tok * hid)[vi]
                                                 : make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int k = 0; k < kUnroll; ++k) {
        const int vi = vb + k * 32 + lane;
        if (vi >= nvec) continue;
        float x[kTok][V];
#pragma unroll
        for (int u = 0; u < kTok; ++u) {
          unpack16(raw[k][u], x[u], static_cast<const TA*>(nullptr));
#pragma unroll
          for (int e = 0; e < V; ++e) ss[u] = fmaf(x[u][e], x[u][e], ss[u]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < H) {
            const float* wp = wg + j * hid + vi * V;
#pragma unroll
            for (int e = 0; e < V; ++e) {
              const float wv = wp[e];
#pragma unroll
              for (int u = 0; u < kTok; ++u) dot[u][j] = fmaf(wv, x[u][e], dot[u][j]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot[u][j] += __shfl_xor_sync(0xffffffffu, dot[u][j], o);
    }
    if (lane < kTok) {
      // lane u writes token tok0 + u (register arrays indexed with a constant)
#pragma unroll
      for (int u = 0; u < kTok; ++u) {
        if (u != lane) continue;
        const long tok = tok0 + u;
        if (tok >= ntok) continue;
        const int b = static_cast<int>(tok / T), t = static_cast<int>(tok % T);
        float a0 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j >= H) continue;
          const int src = layer_mode ? 0 : j;
          const float al = adapter_logit(c, dot[u][src], ss[u], hid, bias ? to_f(bias[src]) : 0.f,
                                         a.offset[b * a.offset_bstride + src]);
          if (j == 0) a0 = al;
          alpha[(static_cast<long>(b) * H + j) * T + t] = layer_mode ? a0 : al;
        }
      }
    }
  }
}

// Decode-shaped variant (one token per sequence): one CTA per (kv-head, b),
// the hidden row and W_h read straight from global memory as 16-byte vectors.
template <typename TA>
__global__ void __launch_bounds__(256) k_decide_proj_row(CacheView c, DecideArgs a, float* alpha) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int src = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
  const int hid = c.hidden;
  constexpr int V = 16 / sizeof(TA);
  const uint4* x = reinterpret_cast<const uint4*>(static_cast<const TA*>(a.hidden) + static_cast<long>(b) * hid);
  const uint4* W = reinterpret_cast<const uint4*>(static_cast<const TA*>(a.W) + static_cast<long>(src) * hid);
  float ss = 0.f, dot = 0.f;
  for (int vi = threadIdx.x; vi < hid / V; vi += blockDim.x) {
    float xv[V], wv[V], gv[V];
    unpack16(x[vi], xv, static_cast<const TA*>(nullptr));
    unpack16(W[vi], wv, static_cast<const TA*>(nullptr));
    unpack16(gamma16<TA>(a.gamma, vi), gv, static_cast<const TA*>(nullptr));
#pragma unroll
    for (int e = 0; e < V; ++e) {
      ss = fmaf(xv[e], xv[e], ss);
      dot = fmaf(wv[e] * gv[e], xv[e], dot);
    }
  }
  __shared__ float red[2][32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) {
    red[0][wid] = ss;
    red[1][wid] = dot;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s2 = 0.f, d2 = 0.f;
    for (int i = 0; i < (blockDim.x >> 5); ++i) {
      s2 += red[0][i];
      d2 += red[1][i];
    }
    const TA* bias = static_cast<const TA*>(a.bias);
    alpha[b * c.Hkv + h] =
        adapter_logit(c, d2, s2, hid, bias ? to_f(bias[src]) : 0.f, a.offset[b * a.offset_bstride + src]);
  }
}

// ---------------------------------------------------------------------------
// The same logits for bf16 activations on the tensor cores: a product of the
// hidden rows [B*T, hidden] with the folded weights (W_h * gamma)^T
// [hidden, Hkv <= 8], N padded to 8.  W * gamma (exact in 16 bits) is held in
// shared memory as a bf16 pair hi + lo, so two mma.sync per k-step give the
// product with fp32 accumulation; the rows' sums of squares come from the A
// fragments already in registers.  Hidden tiles (64 tokens x 64 elements)
// stream through an 8-stage TMA ring (no multicast) fed by a producer warp; a
// persistent grid walks the 64-token tiles.  Consumer warp w takes tokens
// [16 (w % 4), +16) of the even (w < 4) or odd chunks of the hidden size; the
// two halves are added through shared memory at the end of the tile.
// ---------------------------------------------------------------------------
constexpr int kDpTok = 64, kDpK = 128, kDpStages = 4, kDpWarps = 8;  // a stage: two 64-element boxes
// chunks the producer keeps warm in L2 ahead of the ring (the ring is bounded
// by the shared memory the table leaves; the prefetches are not)
constexpr int kDpPrefetch = 8;
static_assert(kDpStages % 2 == 0, "a stage must keep one consumer parity");
constexpr int kDpFillU = 8;  // table items a thread loads before it writes any
constexpr int kDpThreads = (kDpWarps + 1) * 32;

// table row (bf16): the hidden size rounded up to whole chunks (zero-filled,
// so the last chunk's columns past the hidden size read zeros) plus a
// 16-byte pad that keeps the ldmatrix rows on distinct banks
__host__ __device__ inline int dp_wrow(int hid) { return (hid + kDpK - 1) / kDpK * kDpK + 8; }
// byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled TMA tile
__device__ __forceinline__ uint32_t dp_sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}
__host__ __device__ inline size_t dp_smem(int hid) {
  return 1024 + static_cast<size_t>(kDpStages) * kDpTok * 2 * kDpK + 2ull * 8 * dp_wrow(hid) * 2;
}

__global__ void __launch_bounds__(kDpThreads, 1)
    k_decide_proj_tc(CacheView c, int T, DecideArgs a, float* alpha, const __grid_constant__ CUtensorMap hmap) {
  extern __shared__ __align__(1024) unsigned char dp_raw[];
  unsigned char* sb = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dp_raw) + 1023) & ~uintptr_t(1023));
  __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(sb + kDpStages * kDpTok * 2 * kDpK);  // [2][8][wrow]
  __shared__ __align__(8) uint64_t full[kDpStages], empty[kDpStages];
  __shared__ float red[4][6][32];  // odd-chunk halves: acc[4], ss[2] per lane of warps 4..7
  const int H = c.Hkv, hid = c.hidden, wrow = dp_wrow(hid);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long ntok = static_cast<long>(c.B) * T;
  const int ntiles = static_cast<int>((ntok + kDpTok - 1) / kDpTok), nk = (hid + kDpK - 1) / kDpK;
  // chunk q of this CTA: tile blockIdx.x + (q / nk) * gridDim.x, column chunk q % nk
  const int nq = (ntiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                 static_cast<int>(gridDim.x) * nk;
  auto chunk_x = [&](int q) { return (q % nk) * kDpK; };
  auto chunk_y = [&](int q) { return (static_cast<int>(blockIdx.x) + (q / nk) * static_cast<int>(gridDim.x)) * kDpTok; };
  auto issue = [&](int q) {
    const int st = q % kDpStages;
    mbar_expect_tx(&full[st], kDpTok * 2 * kDpK);
    for (int hb = 0; hb < kDpK / 64; ++hb)
      tma_load_2d(sb + st * kDpTok * 2 * kDpK + hb * kDpTok * 128, &hmap, chunk_x(q) + 64 * hb, chunk_y(q), &full[st]);
  };
  auto prefetch = [&](int q) {
    for (int hb = 0; hb < kDpK / 64; ++hb) tma_prefetch_2d(&hmap, chunk_x(q) + 64 * hb, chunk_y(q));
  };
  if (warp == kDpWarps && lane == 0) {
    // the producer sets up the ring and starts it (and the L2 prefetches)
    // before the table is built
    for (int i = 0; i < kDpStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kDpWarps / 2);  // the four warps of the chunk's parity
    }
    fence_mbar_init();
    fence_proxy_async();  // the initialised barriers before this thread's first TMA (async proxy)
    for (int q = 0; q < min(kDpStages, nq); ++q) issue(q);
    for (int q = kDpStages; q < min(kDpStages + kDpPrefetch, nq); ++q) prefetch(q);
  }
  // folded table hi / lo (rows >= H and the pad are zero).  Each thread loads
  // kDpFillU items' W and gamma vectors before it writes any (the table is
  // written through a generic pointer, which would otherwise order every load
  // after the previous item's stores); CTAs start at different items so that
  // they do not all read the same L2 lines at once.
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.W);
  const __nv_bfloat16* gamma = static_cast<const __nv_bfloat16*>(a.gamma);
  const int nvec = hid / 8, rvec = wrow / 8, nitem = 8 * rvec;
  const int rot = static_cast<int>((blockIdx.x * 613u) % static_cast<unsigned>(nitem));
  for (int i0 = tid; i0 < nitem; i0 += kDpThreads * kDpFillU) {
    uint4 wq[kDpFillU], gq[kDpFillU];
    int it[kDpFillU];
#pragma unroll
    for (int u = 0; u < kDpFillU; ++u) {
      int i = i0 + u * kDpThreads;
      it[u] = -1;
      wq[u] = gq[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i >= nitem) continue;
      i += rot;
      if (i >= nitem) i -= nitem;
      it[u] = i;
      const int n = i / rvec, v = i % rvec;
      if (n < H && v < nvec) {
        wq[u] = reinterpret_cast<const uint4*>(W + static_cast<long>(n) * hid)[v];
        gq[u] = gamma16<__nv_bfloat16>(gamma, v);
      }
    }
#pragma unroll
    for (int u = 0; u < kDpFillU; ++u) {
      if (it[u] < 0) continue;
      const int n = it[u] / rvec, v = it[u] % rvec;
      float wv[8], gv[8];
      unpack16(wq[u], wv, static_cast<const __nv_bfloat16*>(nullptr));
      unpack16(gq[u], gv, static_cast<const __nv_bfloat16*>(nullptr));
      uint32_t h4[4], l4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p0 = wv[2 * e] * gv[2 * e], p1 = wv[2 * e + 1] * gv[2 * e + 1];
        const __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
        const float2 hf = __bfloat1622float2(hv);
        h4[e] = *reinterpret_cast<const uint32_t*>(&hv);
        l4[e] = pack_bf16(p0 - hf.x, p1 - hf.y);
      }
      reinterpret_cast<uint4*>(wt + static_cast<long>(n) * wrow)[v] = make_uint4(h4[0], h4[1], h4[2], h4[3]);
      reinterpret_cast<uint4*>(wt + static_cast<long>(8 + n) * wrow)[v] = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    }
  }
  __syncthreads();

  if (warp == kDpWarps) {
    // ---- producer: hidden tiles of this CTA's token tiles ----------------
    if (lane == 0) {
      for (int q = kDpStages; q < nq; ++q) {
        const int st = q % kDpStages, use = q / kDpStages;
        if (!mbar_wait_bounded(&empty[st], (use - 1) & 1)) {
          set_status(c.ctrl, DMS_ST_TIMEOUT);
          return;
        }
        issue(q);
        if (q + kDpPrefetch < nq) prefetch(q + kDpPrefetch);
      }
    }
    return;
  }
  // ---- consumers ----------------------------------------------------------
  const bool layer_mode = c.alpha_per == DMS_ALPHA_PER_LAYER;
  const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(a.bias);
  const int mt = warp & 3, par = warp >> 2;  // token group, chunk parity
  const int mi = lane >> 3, rr = lane & 7;
  // ldmatrix row addresses: A rows of this warp; B = table rows n (hi: matrices 0, 1; lo: 2, 3)
  const int arow = mt * 16 + (mi & 1) * 8 + rr;
  const uint32_t wbase = smem_u32(wt + static_cast<long>((mi >> 1) * 8 + rr) * wrow + (mi & 1) * 8);
  int qbase = 0;  // chunks of the CTA's earlier tiles
  bool ok = true;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, qbase += nk) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float ss[2] = {0.f, 0.f};
    // chunk q goes to the warps of parity q % 2: with an even stage count a
    // stage is always consumed by the same four warps, in order
    for (int kc = par ^ (qbase & 1); kc < nk; kc += 2) {
      const int q = qbase + kc, st = q % kDpStages;
      if (ok && !mbar_wait_bounded(&full[st], (q / kDpStages) & 1)) {
        ok = false;
        if (lane == 0) set_status(c.ctrl, DMS_ST_TIMEOUT);
      }
      if (ok) {
        const uint32_t xs = smem_u32(sb + st * kDpTok * 2 * kDpK);
#pragma unroll
        for (int ks = 0; ks < kDpK / 16; ++ks) {
          uint32_t af[4], bf[4];
          ldmatrix_x4(af[0], af[1], af[2], af[3],
                      xs + (ks / 4) * (kDpTok * 128) + dp_sw128(arow, 2 * (ks % 4) + (mi >> 1)));
          ldmatrix_x4(bf[0], bf[1], bf[2], bf[3], wbase + 2u * static_cast<uint32_t>(kc * kDpK + ks * 16));
          mma_bf16_16816(acc, af, bf);
          mma_bf16_16816(acc, af, bf + 2);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float2 xv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&af[r]));
            ss[r & 1] = fmaf(xv.x, xv.x, fmaf(xv.y, xv.y, ss[r & 1]));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // add the odd-chunk half (warp mt + 4) into warp mt
    if (par == 1) {
#pragma unroll
      for (int e = 0; e < 4; ++e) red[mt][e][lane] = acc[e];
      red[mt][4][lane] = ss[0];
      red[mt][5][lane] = ss[1];
    }
    asm volatile("bar.sync 1, %0;\n" ::"n"(kDpWarps * 32) : "memory");
    if (par == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] += red[mt][e][lane];
      ss[0] += red[mt][4][lane];
      ss[1] += red[mt][5][lane];
      // rows lane/4 and lane/4 + 8 of the group: sums over the 4 lanes of a row
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], 1);
        ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], 2);
      }
      // layer granularity: every head takes head 0's logit (column 0, lane 4 * row)
      float h0[2];
      h0[0] = __shfl_sync(0xffffffffu, acc[0], lane & ~3);
      h0[1] = __shfl_sync(0xffffffffu, acc[2], lane & ~3);
      if (ok) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const long tok = static_cast<long>(tile) * kDpTok + mt * 16 + (lane >> 2) + 8 * r;
          if (tok >= ntok) continue;
          const int b = static_cast<int>(tok / T), t = static_cast<int>(tok % T);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = 2 * (lane & 3) + e;
            if (j >= H) continue;
            const int src = layer_mode ? 0 : j;
            const float dot = layer_mode ? h0[r] : acc[2 * r + e];
            alpha[(static_cast<long>(b) * H + j) * T + t] = adapter_logit(
                c, dot, ss[r], hid, bias ? __bfloat162float(bias[src]) : 0.f, a.offset[b * a.offset_bstride + src]);
          }
        }
      }
    }
    asm volatile("bar.sync 1, %0;\n" ::"n"(kDpWarps * 32) : "memory");  // red is free again
  }
}

cudaError_t launch_decide_proj(const CacheView& c, int T, const DecideArgs& a, float* alpha, const CUtensorMap* hmap,
                               cudaStream_t s) {
  if (T == 1) {
    dim3 grid(c.Hkv, c.B);
    if (c.act_dtype == DMS_BF16)
      k_decide_proj_row<__nv_bfloat16><<<grid, 256, 0, s>>>(c, a, alpha);
    else
      k_decide_proj_row<float><<<grid, 256, 0, s>>>(c, a, alpha);
    return cudaGetLastError();
  }
  const long ntok = static_cast<long>(c.B) * T;
  cudaError_t e;
  if (c.act_dtype == DMS_BF16 && hmap && c.Hkv <= 8) {
    int dev = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    const size_t smem = dp_smem(c.hidden);
    if (smem + 1024 <= static_cast<size_t>(optin)) {
      e = cudaFuncSetAttribute(k_decide_proj_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      const long tiles = (ntok + kDpTok - 1) / kDpTok;
      const int grid = static_cast<int>(min(tiles, static_cast<long>(c.num_sms)));
      k_decide_proj_tc<<<grid, kDpThreads, smem, s>>>(c, T, a, alpha, *hmap);
      return cudaGetLastError();
    }
  }
  const size_t smem = static_cast<size_t>(c.Hkv) * c.hidden * sizeof(float);
  const long want = (ntok + 8 * kTok - 1) / (8 * kTok);
  const int grid = static_cast<int>(min(want, static_cast<long>(c.num_sms)));
  if (c.act_dtype == DMS_BF16) {
    e = cudaFuncSetAttribute(k_decide_proj<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_decide_proj<__nv_bfloat16><<<grid, 256, smem, s>>>(c, T, a, alpha);
  } else {
    e = cudaFuncSetAttribute(k_decide_proj<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_decide_proj<float><<<grid, 256, smem, s>>>(c, T, a, alpha);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Neuron decisions and rotary embedding, one thread per (token, row, i <
// D/2) element pair, in place:
//  1. (neuron source) alpha = x[D-1] * scale - offset for the key of head h or
//     the query of head h*g, read by the thread of pair i = D/2 - 1 of that
//     row; layer granularity takes head 0's value; then the decision element
//     of every head is set to zero;
//  2. (tables given) half-split rotation of every query and key row of the
//     token at position t (prefill), or at the sequence's current position
//     pos_dev[b] (decode, T == 1).
// ---------------------------------------------------------------------------
template <typename TA>
__global__ void k_neuron_rope(CacheView c, int T, const int* pos_dev, TA* q, TA* k, const float* offset, int ostride,
                              int do_alpha, float* alpha, const float* cos_t, const float* sin_t) {
  griddep_wait();
  griddep_launch_dependents();
  const int D = c.D, half = D / 2, g = c.Hq / c.Hkv;
  const bool key = c.alpha_source == DMS_ALPHA_KEY_NEURON;
  // with rotary tables every (token, row, i < D/2) pair, else only the
  // decision neuron of each head (its pair i = D/2 - 1)
  const int nrow = cos_t ? c.Hq + c.Hkv : c.Hkv;
  const int npair = cos_t ? half : 1;
  const long total = static_cast<long>(c.B) * T * nrow * npair;
  for (long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int i = cos_t ? static_cast<int>(idx % half) : half - 1;
    const long rt = idx / npair;
    int r = static_cast<int>(rt % nrow);
    const long tok = rt / nrow;
    if (!cos_t) r = key ? c.Hq + r : r * g;  // the neuron rows only
    const int b = static_cast<int>(tok / T), t = static_cast<int>(tok % T);
    TA* row = r < c.Hq ? q + (tok * c.Hq + r) * D : k + (tok * c.Hkv + (r - c.Hq)) * D;
    float x0 = to_f(row[i]), x1 = to_f(row[i + half]);
    // the decision neuron (the last element of each key, or of the first query
    // head of each group) is read, then zeroed, before the rotation
    const bool neuron_row = key ? r >= c.Hq : (r < c.Hq && r % g == 0);
    if (do_alpha && neuron_row && i == half - 1) {
      const int h = key ? r - c.Hq : r / g;
      if (c.alpha_per == DMS_ALPHA_PER_LAYER) {
        if (h == 0) {
          const float a = fmaf(x1, c.alpha_scale, -offset[b * ostride]);
          for (int hh = 0; hh < c.Hkv; ++hh) alpha[(static_cast<long>(b) * c.Hkv + hh) * T + t] = a;
        }
      } else {
        alpha[(static_cast<long>(b) * c.Hkv + h) * T + t] = fmaf(x1, c.alpha_scale, -offset[b * ostride + h]);
      }
      x1 = 0.f;
    }
    if (cos_t) {
      const int p = pos_dev ? pos_dev[b] + t : t;
      const float cv = cos_t[static_cast<long>(p) * half + i], sv = sin_t[static_cast<long>(p) * half + i];
      // the rotation in fp64, rounded once into the activation dtype
      double y0, y1;
      rotate64(x0, x1, cv, sv, y0, y1);
      row[i] = from_f64<TA>(y0);
      row[i + half] = from_f64<TA>(y1);
    } else {
      row[i + half] = from_f<TA>(x1);
    }
  }
}

// Four consecutive pairs (i .. i+3 < D/2) of one row per thread and step: the
// same arithmetic as above with 8- or 16-byte accesses (rotary tables given;
// rows and tables 16-byte aligned).
template <typename TA>
__device__ __forceinline__ void ld4(const TA* p, float* f);
template <>
__device__ __forceinline__ void ld4<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  f[0] = a.x;
  f[1] = a.y;
  f[2] = b.x;
  f[3] = b.y;
}
template <>
__device__ __forceinline__ void ld4<float>(const float* p, float* f) {
  const float4 u = *reinterpret_cast<const float4*>(p);
  f[0] = u.x;
  f[1] = u.y;
  f[2] = u.z;
  f[3] = u.w;
}
template <typename TA>
__device__ __forceinline__ void st4(TA* p, const float* f);
template <>
__device__ __forceinline__ void st4<__nv_bfloat16>(__nv_bfloat16* p, const float* f) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
}
template <>
__device__ __forceinline__ void st4<float>(float* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}

// An fp64 rotation result narrowed to fp32 so that st4's conversion into the
// activation dtype rounds it exactly once: bf16 rows keep it rounded to odd
// (st4 then rounds to nearest even), fp32 rows round it to nearest even here.
template <typename TA>
__device__ __forceinline__ float narrow_f64(double x);
template <>
__device__ __forceinline__ float narrow_f64<float>(double x) { return __double2float_rn(x); }
template <>
__device__ __forceinline__ float narrow_f64<__nv_bfloat16>(double x) { return f64_to_f32_odd(x); }

template <typename TA>
__global__ void k_neuron_rope4(CacheView c, int T, const int* pos_dev, TA* q, TA* k, const float* offset, int ostride,
                               int do_alpha, float* alpha, const float* cos_t, const float* sin_t) {
  griddep_wait();
  griddep_launch_dependents();
  const int D = c.D, half = D / 2, nq = half / 4, g = c.Hq / c.Hkv;
  const bool key = c.alpha_source == DMS_ALPHA_KEY_NEURON;
  const int nrow = c.Hq + c.Hkv;
  const long total = static_cast<long>(c.B) * T * nrow * nq;
  for (long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(idx % nq) * 4;
    const long rt = idx / nq;
    const int r = static_cast<int>(rt % nrow);
    const long tok = rt / nrow;
    const int b = static_cast<int>(tok / T), t = static_cast<int>(tok % T);
    TA* row = r < c.Hq ? q + (tok * c.Hq + r) * D : k + (tok * c.Hkv + (r - c.Hq)) * D;
    float x0[4], x1[4], cv[4], sv[4];
    ld4<TA>(row + i, x0);
    ld4<TA>(row + i + half, x1);
    const int p = pos_dev ? pos_dev[b] + t : t;
    ld4<float>(cos_t + static_cast<long>(p) * half + i, cv);
    ld4<float>(sin_t + static_cast<long>(p) * half + i, sv);
    // the decision neuron (pair half - 1: the last element of the row) is
    // read, then zeroed, before the rotation
    const bool neuron_row = key ? r >= c.Hq : (r < c.Hq && r % g == 0);
    if (do_alpha && neuron_row && i + 3 == half - 1) {
      const int h = key ? r - c.Hq : r / g;
      if (c.alpha_per == DMS_ALPHA_PER_LAYER) {
        if (h == 0) {
          const float a = fmaf(x1[3], c.alpha_scale, -offset[b * ostride]);
          for (int hh = 0; hh < c.Hkv; ++hh) alpha[(static_cast<long>(b) * c.Hkv + hh) * T + t] = a;
        }
      } else {
        alpha[(static_cast<long>(b) * c.Hkv + h) * T + t] = fmaf(x1[3], c.alpha_scale, -offset[b * ostride + h]);
      }
      x1[3] = 0.f;
    }
    float y0[4], y1[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // the rotation in fp64, narrowed so that st4's rounding into the
      // activation dtype is the only rounding of the exact rotation's fp64 value
      double r0, r1;
      rotate64(x0[e], x1[e], cv[e], sv[e], r0, r1);
      y0[e] = narrow_f64<TA>(r0);
      y1[e] = narrow_f64<TA>(r1);
    }
    st4<TA>(row + i, y0);
    st4<TA>(row + i + half, y1);
  }
}

// bf16 rows, large launches (prefill): one thread per (token, eight
// consecutive pairs i .. i+7 < D/2).  The thread loads its cos/sin entries
// once and walks the token's Hq + Hkv rows kRopeRows at a time, issuing all of
// a group's loads before the first rotation; 32-bit indices (the launcher
// checks that the item count fits).  The same arithmetic as above.
constexpr int kRopeRows = 4;

__global__ void __launch_bounds__(256, 3) k_neuron_rope8(CacheView c, int T, const int* pos_dev, __nv_bfloat16* q,
                                                      __nv_bfloat16* k, const float* offset, int ostride,
                                                      int do_alpha, float* alpha, const float* cos_t,
                                                      const float* sin_t) {
  griddep_wait();
  griddep_launch_dependents();
  const int D = c.D, half = D / 2, nq = half / 8, g = c.Hq / c.Hkv;
  const bool key = c.alpha_source == DMS_ALPHA_KEY_NEURON;
  const int nrow = c.Hq + c.Hkv;
  const int total = c.B * T * nq;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += gridDim.x * blockDim.x) {
    const int i = (idx % nq) * 8, tok = idx / nq;
    const int b = tok / T, t = tok - b * T;
    const long p = static_cast<long>(pos_dev ? pos_dev[b] + t : t) * half + i;
    float cv[8], sv[8];
    {
      const float4 c0 = *reinterpret_cast<const float4*>(cos_t + p), c1 = *reinterpret_cast<const float4*>(cos_t + p + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(sin_t + p), s1 = *reinterpret_cast<const float4*>(sin_t + p + 4);
      cv[0] = c0.x, cv[1] = c0.y, cv[2] = c0.z, cv[3] = c0.w, cv[4] = c1.x, cv[5] = c1.y, cv[6] = c1.z, cv[7] = c1.w;
      sv[0] = s0.x, sv[1] = s0.y, sv[2] = s0.z, sv[3] = s0.w, sv[4] = s1.x, sv[5] = s1.y, sv[6] = s1.z, sv[7] = s1.w;
    }
    __nv_bfloat16* qrow = q + static_cast<long>(tok) * c.Hq * D + i;
    __nv_bfloat16* krow = k + static_cast<long>(tok) * c.Hkv * D + i;
    for (int r0 = 0; r0 < nrow; r0 += kRopeRows) {
      uint4 x0[kRopeRows], x1[kRopeRows];
#pragma unroll
      for (int u = 0; u < kRopeRows; ++u) {
        const int r = r0 + u;
        if (r >= nrow) continue;
        const __nv_bfloat16* row = r < c.Hq ? qrow + r * D : krow + (r - c.Hq) * D;
        x0[u] = *reinterpret_cast<const uint4*>(row);
        x1[u] = *reinterpret_cast<const uint4*>(row + half);
      }
#pragma unroll
      for (int u = 0; u < kRopeRows; ++u) {
        const int r = r0 + u;
        if (r >= nrow) continue;
        float a0[8], a1[8];
        unpack16(x0[u], a0, static_cast<const __nv_bfloat16*>(nullptr));
        unpack16(x1[u], a1, static_cast<const __nv_bfloat16*>(nullptr));
        // the decision neuron (pair half - 1: the last element of the row) is
        // read, then zeroed, before the rotation
        const bool neuron_row = key ? r >= c.Hq : (r < c.Hq && r % g == 0);
        if (do_alpha && neuron_row && i + 7 == half - 1) {
          const int h = key ? r - c.Hq : r / g;
          if (c.alpha_per == DMS_ALPHA_PER_LAYER) {
            if (h == 0) {
              const float av = fmaf(a1[7], c.alpha_scale, -offset[b * ostride]);
              for (int hh = 0; hh < c.Hkv; ++hh) alpha[(static_cast<long>(b) * c.Hkv + hh) * T + t] = av;
            }
          } else {
            alpha[(static_cast<long>(b) * c.Hkv + h) * T + t] = fmaf(a1[7], c.alpha_scale, -offset[b * ostride + h]);
          }
          a1[7] = 0.f;
        }
        uint32_t y0[4], y1[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // the rotation in fp64, rounded once into bf16
          const int j = 2 * e;
          double r0a, r1a, r0b, r1b;
          rotate64(a0[j], a1[j], cv[j], sv[j], r0a, r1a);
          rotate64(a0[j + 1], a1[j + 1], cv[j + 1], sv[j + 1], r0b, r1b);
          y0[e] = pack_bf16_f64(r0a, r0b);
          y1[e] = pack_bf16_f64(r1a, r1b);
        }
        __nv_bfloat16* row = r < c.Hq ? qrow + r * D : krow + (r - c.Hq) * D;
        *reinterpret_cast<uint4*>(row) = make_uint4(y0[0], y0[1], y0[2], y0[3]);
        *reinterpret_cast<uint4*>(row + half) = make_uint4(y1[0], y1[1], y1[2], y1[3]);
      }
    }
  }
}

// A launch of kern<<<grid, 256, 0, s>>>, as a programmatic dependent of the
// previous kernel on the stream when pdl is set.
template <typename... KArgs, typename... Args>
static cudaError_t launch_rope_kernel(void (*kern)(KArgs...), int grid, cudaStream_t s, bool pdl, Args... args) {
  if (pdl) return launch_dependent(kern, dim3(grid), dim3(256), 0, s, args...);
  kern<<<grid, 256, 0, s>>>(static_cast<KArgs>(args)...);
  return cudaGetLastError();
}

cudaError_t launch_neuron_rope(const CacheView& c, int T, const int* pos_dev, void* q, void* k, const float* offset,
                               int offset_bstride, bool do_alpha, float* alpha, const float* cos_t,
                               const float* sin_t, cudaStream_t s, bool pdl) {
  const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(cos_t) | reinterpret_cast<uintptr_t>(sin_t);
  const int da = do_alpha ? 1 : 0;
  // large bf16 launches: one thread per (token, 8 pairs), rows walked in groups
  const long total8 = static_cast<long>(c.B) * T * (c.D / 16);
  if (cos_t && (al & 15) == 0 && (c.D / 2) % 8 == 0 && c.act_dtype == DMS_BF16 &&
      total8 >= static_cast<long>(c.num_sms) * 256 && total8 < (1L << 30)) {
    const int grid8 = static_cast<int>(min((total8 + 255) / 256, static_cast<long>(c.num_sms) * 3));
    return launch_rope_kernel(k_neuron_rope8, grid8, s, pdl, c, T, pos_dev, static_cast<__nv_bfloat16*>(q),
                              static_cast<__nv_bfloat16*>(k), offset, offset_bstride, da, alpha, cos_t, sin_t);
  }
  if (cos_t && (al & 15) == 0 && (c.D / 2) % 4 == 0) {
    const long total4 = static_cast<long>(c.B) * T * (c.Hq + c.Hkv) * (c.D / 8);
    const int grid4 = static_cast<int>(max(1L, min((total4 + 255) / 256, static_cast<long>(c.num_sms) * 16)));
    if (c.act_dtype == DMS_BF16)
      return launch_rope_kernel(k_neuron_rope4<__nv_bfloat16>, grid4, s, pdl, c, T, pos_dev,
                                static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k), offset, offset_bstride,
                                da, alpha, cos_t, sin_t);
    return launch_rope_kernel(k_neuron_rope4<float>, grid4, s, pdl, c, T, pos_dev, static_cast<float*>(q),
                              static_cast<float*>(k), offset, offset_bstride, da, alpha, cos_t, sin_t);
  }
  const long total = static_cast<long>(c.B) * T * (cos_t ? (c.Hq + c.Hkv) * (c.D / 2) : c.Hkv);
  const int grid = static_cast<int>(max(1L, min((total + 255) / 256, static_cast<long>(c.num_sms) * 16)));
  if (c.act_dtype == DMS_BF16)
    return launch_rope_kernel(k_neuron_rope<__nv_bfloat16>, grid, s, pdl, c, T, pos_dev,
                              static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k), offset, offset_bstride,
                              da, alpha, cos_t, sin_t);
  return launch_rope_kernel(k_neuron_rope<float>, grid, s, pdl, c, T, pos_dev, static_cast<float*>(q),
                            static_cast<float*>(k), offset, offset_bstride, da, alpha, cos_t, sin_t);
}

}  // namespace dms
