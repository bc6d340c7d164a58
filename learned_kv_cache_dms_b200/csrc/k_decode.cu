// Decode step: append with delayed eviction, then split-K grouped attention
// over each head's compact retained slots.
#include "decode_common.cuh"

namespace dms {


// ---------------------------------------------------------------------------
// Append of token t for every (b, h) of one layer, one CTA per (b, h):
//   if t >= w and the token t - w (ring[t % w]) was marked for eviction, the new
//   token overwrites its slot in place; else it takes slot count++, and a page
//   is granted from the ascending counter when that slot starts a page
//   ([DMS-Qwen3], inference mode with the paged KV cache; [FastDMS], decode
//   kernel: per-step keep/evict, sliding retention window, compact append).
// The decision is the head's plan for position t (slot, flags, count and pages
// before the append, written by the step before); new pages are numbered from
// the counter plus the head's rank among the heads needing one, i.e. in (b, h)
// row-major order (every sequence is at the same position).  The CTA writes the
// K/V row (FP8: re-encodes the page when the new row raises its scale, every
// thread of the CTA taking part), the head's state and the plan of position
// t + 1; the grid's last CTA advances the page counter and the positions.
// With `fuse_decide` the CTA first computes its head's adapter decision logit
// (RMSNorm over the hidden row, one dot product) and writes it to `alpha`.
// ---------------------------------------------------------------------------
constexpr int kAppendThreads = 128;
static_assert(kAppendThreads == kThreads, "fp8_append_row reduces over kThreads threads");

template <typename TA, bool FP8>
__global__ void __launch_bounds__(kAppendThreads) k_decode_append(CacheView c, int layer, const TA* k, const TA* v,
                                                                  float* alpha, DecideArgs da, int fuse_decide) {
  __shared__ int s_red[32];
  __shared__ float s_f[2][kAppendThreads / 32];
  __shared__ int s_last;
  const int BH = c.B * c.Hkv, bh = blockIdx.x;
  const int b = bh / c.Hkv, h = bh % c.Hkv;
  const long lbase = static_cast<long>(layer) * BH, li = lbase + bh;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, w = c.w, P = c.P, D = c.D;
  // every read of this CTA's state first (one round trip; the plan needs t)
  const int t = c.pos[layer * c.B + b];
  const int next_page0 = c.ctrl[CTRL_NEXT_PAGE];
  const int ring_next = (t + 1 >= w) ? c.ring[li * w + (t + 1) % w] : 0;
  const int4 pl = *plan_at(c, li, t);
  const int hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;

  // decision logit of this head (layer granularity: head 0's row of W)
  float a_dec = 0.f;
  if (fuse_decide) {
    constexpr int V = 16 / sizeof(TA);
    const int hid = c.hidden, nvec = hid / V;
    const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const TA*>(da.hidden) + static_cast<long>(b) * hid);
    const uint4* wr = reinterpret_cast<const uint4*>(static_cast<const TA*>(da.W) + static_cast<long>(hs) * hid);
    float ss = 0.f, dot = 0.f;
#pragma unroll 4
    for (int vi = tid; vi < nvec; vi += kAppendThreads) {
      const uint4 xu = xr[vi], wu = wr[vi], gu = gamma16<TA>(da.gamma, vi);
      float x[V], wv[V], gv[V];
      unpack16(xu, x, static_cast<const TA*>(nullptr));
      unpack16(wu, wv, static_cast<const TA*>(nullptr));
      unpack16(gu, gv, static_cast<const TA*>(nullptr));
#pragma unroll
      for (int e = 0; e < V; ++e) {
        ss = fmaf(x[e], x[e], ss);
        dot = fmaf(wv[e] * gv[e], x[e], dot);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      dot += __shfl_xor_sync(0xffffffffu, dot, o);
    }
    if (lane == 0) {
      s_f[0][wid] = ss;
      s_f[1][wid] = dot;
    }
    __syncthreads();
    if (tid == 0) {
      float s2 = 0.f, d2 = 0.f;
      for (int i = 0; i < kAppendThreads / 32; ++i) {
        s2 += s_f[0][i];
        d2 += s_f[1][i];
      }
      const TA* bias = static_cast<const TA*>(da.bias);
      a_dec = adapter_logit(c, d2, s2, hid, bias ? to_f(bias[hs]) : 0.f, da.offset[b * da.offset_bstride + hs]);
      alpha[b * c.Hkv + h] = a_dec;
    }
    __syncthreads();
  }

  // rank among the lower heads needing a new page (their plans for t)
  const int flags = pl.y, slot = pl.x, cnt = pl.z, have = pl.w;
  int id = -1;
  bool ok = !(flags & 4);
  if (ok && (flags & 2)) {
    int n_before = 0;
    for (int i = tid; i < bh; i += kAppendThreads) n_before += (plan_at(c, lbase + i, t)->y & 2) ? 1 : 0;
    int tot;  // lower heads needing a page
    block_exclusive_scan(n_before, s_red, &tot);
    id = next_page0 + tot;
    if (id >= c.pool_pages || have >= c.maxp) ok = false;
  } else if (ok) {
    id = c.page_table[li * c.maxp + slot / P];
  }
  const int cnt_new = (ok && !(flags & 1)) ? cnt + 1 : cnt, np_new = (ok && (flags & 2)) ? have + 1 : have;

  if (ok) {
    const long dst_row = static_cast<long>(id) * P + slot % P;
    const TA* ksrc = k + static_cast<long>(bh) * D;
    const TA* vsrc = v + static_cast<long>(bh) * D;
    if (!FP8) {
      const int cpr = D * static_cast<int>(sizeof(TA)) / 16;
      if (tid < cpr) {
        reinterpret_cast<uint4*>(static_cast<TA*>(c.k_pool) + dst_row * D)[tid] =
            reinterpret_cast<const uint4*>(ksrc)[tid];
        reinterpret_cast<uint4*>(static_cast<TA*>(c.v_pool) + dst_row * D)[tid] =
            reinterpret_cast<const uint4*>(vsrc)[tid];
      }
    } else {
      const int rows = min(P, cnt_new - (slot / P) * P);  // rows in use in that page after the append
      const long pb = static_cast<long>(id) * P * D;
      fp8_append_kv(tid < D ? to_f(ksrc[tid]) : 0.f, tid < D ? to_f(vsrc[tid]) : 0.f,
                    static_cast<uint8_t*>(c.k_pool) + pb, static_cast<uint8_t*>(c.v_pool) + pb, c.k_scale + id,
                    c.v_scale + id, c.k_scale[id], c.v_scale[id], slot % P, rows, D, &s_f[0][0]);
    }
  }
  if (tid == 0) {
    if (ok) {
      if (flags & 2) {
        c.page_table[li * c.maxp + have] = id;
        c.npages[li] = np_new;
      }
      if (!(flags & 1)) c.count[li] = cnt_new;
      const float a = fuse_decide ? a_dec : alpha[b * c.Hkv + hs];
      const bool evict = shifted_mark(c, li, t, !c.disable && a > 0.0f);
      c.slot_pos[li * c.cap + slot] = t;
      c.ring[li * w + t % w] = slot | (evict ? static_cast<int>(RING_EVICT) : 0);
    } else {
      set_status(c.ctrl, (flags & 4) ? DMS_ST_CAPACITY : DMS_ST_POOL_EXHAUSTED);
    }
    // the plan of position t + 1 from the values just written
    *plan_at(c, li, t + 1) = make_plan(ring_next, t + 1, cnt_new, np_new, c);
    // the grid's last CTA advances the page counter and the positions (every
    // CTA has read them by the time it counts itself)
    s_last = count_step(c, ok && (flags & 2) ? 1 : 0, BH, next_page0) ? 1 : 0;
  }
  __syncthreads();
  if (s_last) advance_positions(c, layer, tid, kAppendThreads);
}

template <typename TA, bool FP8>
static cudaError_t launch_append_t(const CacheView& c, int layer, const void* k, const void* v, float* alpha,
                                   const DecideArgs* da, cudaStream_t s) {
  DecideArgs none{};
  k_decode_append<TA, FP8><<<c.B * c.Hkv, kAppendThreads, 0, s>>>(c, layer, static_cast<const TA*>(k),
                                                                  static_cast<const TA*>(v), alpha, da ? *da : none,
                                                                  da ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_decode_append(const CacheView& c, int layer, const void* k, const void* v, float* alpha,
                                 const DecideArgs* fused_decide, int num_sms, cudaStream_t s) {
  (void)num_sms;
  if (c.kv_dtype == DMS_FP8_E4M3) return launch_append_t<__nv_bfloat16, true>(c, layer, k, v, alpha, fused_decide, s);
  if (c.kv_dtype == DMS_BF16) return launch_append_t<__nv_bfloat16, false>(c, layer, k, v, alpha, fused_decide, s);
  return launch_append_t<float, false>(c, layer, k, v, alpha, fused_decide, s);
}

// ---------------------------------------------------------------------------
// fp32 decode attention (CUDA cores, one warp per query head, no split).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) k_decode_attn_f32(CacheView c, int layer, const float* q, float* o) {
  const int hq = blockIdx.x, b = blockIdx.y, lane = threadIdx.x;
  const int g = c.Hq / c.Hkv, h = hq / g, D = c.D, per = D / 32;
  const long lbh = (static_cast<long>(layer) * c.B + b) * c.Hkv + h;
  const int cnt = c.count[lbh];
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  float qv[4], acc[4];
  for (int e = 0; e < per; ++e) {
    qv[e] = q[(static_cast<long>(b) * c.Hq + hq) * D + lane * per + e] * scale;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const float* kp = static_cast<const float*>(c.k_pool);
  const float* vp = static_cast<const float*>(c.v_pool);
  for (int s = 0; s < cnt; ++s) {
    const int id = c.page_table[lbh * c.maxp + s / c.P];
    const long row = (static_cast<long>(id) * c.P + s % c.P) * D + lane * per;
    float x = 0.f;
    for (int e = 0; e < per; ++e) x = fmaf(qv[e], kp[row + e], x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    const float mn = fmaxf(m, x);
    const float corr = expf(m - mn), p = expf(x - mn);
    l = l * corr + p;
    for (int e = 0; e < per; ++e) acc[e] = acc[e] * corr + p * vp[row + e];
    m = mn;
  }
  for (int e = 0; e < per; ++e) o[(static_cast<long>(b) * c.Hq + hq) * D + lane * per + e] = acc[e] / l;
}

// ---------------------------------------------------------------------------
// bf16 / FP8 split-K decode attention with global partials ([FastDMS],
// attention scoring: split-K grouped compact decode attention over
// variable-length per-head live spans), used by dms_decode_attention.
//
// Every CTA derives the same work partition from the heads' retained counts
// and walks its items (chunks of one head's slots inside one page) in grid
// stride.  Sub-tiles of 64 slots are staged by TMA (16-row boxes, no
// multicast) into a ring of shared-memory stages; 4 warps take 16 slots each
// and run QK^T and PV on mma.sync with the g query heads of the KV head as the
// M dimension (padded to 16), so every K/V byte is read once per step.  Each
// item leaves an unnormalised partial (acc, running max, running sum, log2
// domain) in global scratch; the CTA that finishes a head's last item (per-head
// arrival counter) merges the head's partials and writes its output rows.
// bf16 pages arrive with the 128-byte swizzle; FP8 pages arrive unswizzled and
// are widened to bf16 codes (exact) in shared memory, their page scale applied
// to the scores (K) and to the partial (V).
// ---------------------------------------------------------------------------
template <int D, bool FP8>
__global__ void __launch_bounds__(kThreads) k_decode_attn(CacheView c, int layer, const __nv_bfloat16* q,
                                                         __nv_bfloat16* o, int target_items,
                                                         const __grid_constant__ CUtensorMap kmap,
                                                         const __grid_constant__ CUtensorMap vmap) {
  using S = DecodeSmem<D, FP8>;
  constexpr int KS = D / 16, NT = D / 8, MLD = D + 2;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sbase =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* stage_buf = sbase;                             // kStages * STAGE
  unsigned char* conv_buf = sbase + kStages * S::STAGE;         // FP8: widened K, V
  float* merge = reinterpret_cast<float*>(conv_buf + S::CONV);  // [4 warps][g rows][D + 2]
  const int g = c.Hq / c.Hkv;
  const int BH = c.B * c.Hkv;
  int* s_off = reinterpret_cast<int*>(merge + 4 * g * MLD);  // [BH + 1] first work item of each head
  int* s_cnt = s_off + BH + 1;                               // [BH] retained slots of each head
  float* wbuf = reinterpret_cast<float*>(s_cnt + BH);        // [2 * kCombineChunk + 32] combine staging
  __shared__ uint64_t full_bar[kStages];
  __shared__ StageMeta meta[kStages];
  __shared__ int s_abort, s_last, s_have;
  __shared__ int s_red[32][4];

  const int tid = threadIdx.x;
  const long lbase = static_cast<long>(layer) * BH;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&full_bar[i], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  const int C = decode_partition(c.count + lbase, BH, c.P, target_items, s_cnt, s_off, s_red);
  const int nitems = s_off[BH];

  // producer iterator (thread 0 only)
  int p_item = blockIdx.x, p_sub = 0, p_bh = 0;
  auto produce = [&](int stage) -> bool {
    while (p_item < nitems) {
      while (s_off[p_bh + 1] <= p_item) ++p_bh;  // items are visited in increasing order
      const int s0 = (p_item - s_off[p_bh]) * C;
      const int len = min(s_cnt[p_bh], s0 + C) - s0;
      if (p_sub < len) {
        const int slot0 = s0 + p_sub;
        const int page = c.page_table[(lbase + p_bh) * c.maxp + slot0 / c.P];
        StageMeta& m = meta[stage];
        m.item = p_item;
        m.bh = p_bh;
        m.s0 = s0;
        m.sub = p_sub;
        m.rows = min(kSub, len - p_sub);
        m.page = page;
        m.last = (p_sub + kSub >= len) ? 1 : 0;
        issue_subtile<D, FP8>(stage_buf + stage * S::STAGE, &kmap, &vmap, page * c.P + slot0 % c.P, m.rows,
                              &full_bar[stage]);
        p_sub += kSub;
        return true;
      }
      p_item += gridDim.x;
      p_sub = 0;
    }
    return false;
  };

  int produced = 0;
  if (tid == 0)
    for (int st = 0; st < kStages; ++st)
      if (produce(st)) ++produced;

  uint32_t qa[KS][4];
  float acc[NT][4];
  float mrow[2], lrow[2];
  int cur_item = -1;
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));

  for (int n = 0;; ++n) {
    __syncthreads();
    if (s_abort) break;
    const int stage = n % kStages;
    if (tid == 0) s_have = (n < produced) ? 1 : 0;
    __syncthreads();
    if (!s_have) break;
    if (!mbar_wait_bounded(&full_bar[stage], (n / kStages) & 1)) {
      if (tid == 0) {
        set_status(c.ctrl, DMS_ST_TIMEOUT);
        s_abort = 1;
      }
      __syncthreads();
      break;
    }
    const StageMeta m = meta[stage];
    const int bh = m.bh, b = bh / c.Hkv, h = bh % c.Hkv;
    const unsigned char* kt = stage_buf + stage * S::STAGE;
    if (FP8) {
      widen_fp8_subtile<D>(kt, conv_buf);
      __syncthreads();
      kt = conv_buf;
    }
    const unsigned char* vt = kt + (FP8 ? S::TILE_BF16 : S::TILE_RAW);
    if (m.item != cur_item) {
      cur_item = m.item;
      load_q_frags<D>(q + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D, g, qa);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      mrow[0] = mrow[1] = -INFINITY;
      lrow[0] = lrow[1] = 0.f;
    }
    const int warp = tid >> 5;
    if (warp * 16 < m.rows) {
      const float kscale = FP8 ? c.k_scale[m.page] : 1.0f;
      const float vscale = FP8 ? c.v_scale[m.page] : 1.0f;
      warp_tile<D>(kt, vt, m.rows, -1, kscale * sl2, vscale, qa, acc, mrow, lrow);
    }
    __syncthreads();  // every warp is done with this stage (and with conv_buf)
    if (tid == 0 && produce(stage)) ++produced;

    if (m.last) {
      warp_state_to_smem<D>(merge, warp, g, acc, mrow, lrow);
      __syncthreads();
      merge_to_global<D>(merge, 4, g, 1.0f, c.part_acc, c.part_ml, m.item);
      cur_item = -1;
      // the last CTA to finish one of this head's items merges the head
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        const int nh = s_off[bh + 1] - s_off[bh];
        s_last = (atomicAdd(&c.head_done[bh], 1) == nh - 1) ? 1 : 0;
      }
      __syncthreads();
      if (s_last) {
        __threadfence();
        combine_head<D>(c.part_acc, c.part_ml, g, s_off[bh], s_off[bh + 1],
                        o + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D, wbuf);
        if (tid == 0) c.head_done[bh] = 0;
      }
    }
  }
}

template <int D, bool FP8>
static cudaError_t launch_attn(const CacheView& c, int layer, const void* q, void* o, const CUtensorMap* kmap,
                               const CUtensorMap* vmap, int num_sms, cudaStream_t s) {
  using S = DecodeSmem<D, FP8>;
  const int g = c.Hq / c.Hkv;
  const size_t smem = 1024 + kStages * S::STAGE + S::CONV + 4 * g * (D + 2) * sizeof(float) +
                      (2 * static_cast<size_t>(c.B) * c.Hkv + 1) * sizeof(int) +
                      (2 * kCombineChunk + 32) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_decode_attn<D, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = 2 * num_sms;
  k_decode_attn<D, FP8><<<grid, kThreads, smem, s>>>(c, layer, static_cast<const __nv_bfloat16*>(q),
                                                     static_cast<__nv_bfloat16*>(o), min(num_sms, 160), *kmap, *vmap);
  return cudaGetLastError();
}

cudaError_t launch_decode_attention(const CacheView& c, int layer, const void* q, void* o, const CUtensorMap* kmap,
                                    const CUtensorMap* vmap, int num_sms, cudaStream_t s) {
  if (c.kv_dtype == DMS_F32) {
    dim3 grid(c.Hq, c.B);
    k_decode_attn_f32<<<grid, 32, 0, s>>>(c, layer, static_cast<const float*>(q), static_cast<float*>(o));
    return cudaGetLastError();
  }
  if (!kmap || !vmap) return cudaErrorInvalidValue;
  if (c.kv_dtype == DMS_FP8_E4M3)
    return c.D == 64 ? launch_attn<64, true>(c, layer, q, o, kmap, vmap, num_sms, s)
                     : launch_attn<128, true>(c, layer, q, o, kmap, vmap, num_sms, s);
  return c.D == 64 ? launch_attn<64, false>(c, layer, q, o, kmap, vmap, num_sms, s)
                   : launch_attn<128, false>(c, layer, q, o, kmap, vmap, num_sms, s);
}

}  // namespace dms

