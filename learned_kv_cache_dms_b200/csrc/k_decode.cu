// Decode step: append with delayed eviction, then split-K grouped attention
// over each head's compact retained slots.
#include "decode_common.cuh"

namespace dms {

#ifdef DMS_TRACE
__device__ unsigned long long g_dms_trace[2 * kTraceCtas * kTraceSlots];
#endif

// ---------------------------------------------------------------------------
// Append of token t for every (b, h) of one layer, in one CTA so that page
// grants follow (b, h) row-major order without inter-CTA ordering:
//   if t >= w and the token t - w (ring[t % w]) was marked for eviction, the new
//   token overwrites its slot in place; else it takes slot count++, and a page
//   is granted from the ascending counter when that slot starts a page
//   ([DMS-Qwen3], inference mode with the paged KV cache; [FastDMS], decode
//   kernel: per-step keep/evict, sliding retention window, compact append).
// The same CTA then writes the K/V rows (FP8: re-encodes the page when the new
// row raises its scale).
// With `fuse_decide` the CTA first computes the adapter's decision logits of
// the new tokens (RMSNorm over the hidden row, one dot product per head, one
// warp per dot product) and writes them to `alpha`.
// ---------------------------------------------------------------------------
template <typename TA, bool FP8>
__global__ void __launch_bounds__(1024) k_decode_append(CacheView c, int layer, const TA* k, const TA* v,
                                                       float* alpha, DecideArgs da, int fuse_decide) {
  extern __shared__ int sh[];
  __shared__ int tmp[32];
  const int BH = c.B * c.Hkv;
  int* s_slot = sh;          // slot written by head i (-1: dropped)
  int* s_id = sh + BH;       // page id holding that slot
  int* s_rows = sh + 2 * BH; // rows in use in that page after the append
  const long lbase = static_cast<long>(layer) * BH;
  const int tid = threadIdx.x, bd = blockDim.x, w = c.w, P = c.P;
  const int lane = tid & 31, wid = tid >> 5, nwarp = bd >> 5;
  int next = c.ctrl[CTRL_NEXT_PAGE];
  DMS_TRACE_MARK(1, 0);

  // Phase 0 (optional): decision logits of the new tokens, one warp per
  // (b, h): the mean square of the hidden row and the dot product with
  // W_h * gamma in one pass, four 16-byte vectors of each operand in flight.
  if (fuse_decide) {
    constexpr int V = 16 / sizeof(TA);
    const int hid = c.hidden, nvec = hid / V;
    const TA* hs = static_cast<const TA*>(da.hidden);
    const TA* Wt = static_cast<const TA*>(da.W);
    const TA* gm = static_cast<const TA*>(da.gamma);
    const TA* bias = static_cast<const TA*>(da.bias);
    const bool layer_mode = c.alpha_per == DMS_ALPHA_PER_LAYER;
    const int nh = layer_mode ? 1 : c.Hkv;
    for (int idx = wid; idx < c.B * nh; idx += nwarp) {
      const int b = idx / nh, h = idx % nh;
      const uint4* xr = reinterpret_cast<const uint4*>(hs + static_cast<long>(b) * hid);
      const uint4* wr = reinterpret_cast<const uint4*>(Wt + static_cast<long>(h) * hid);
      const uint4* gr = reinterpret_cast<const uint4*>(gm);
      float ss = 0.f, dot = 0.f;
#pragma unroll 4
      for (int vi = lane; vi < nvec; vi += 32) {
        const uint4 xu = xr[vi], wu = wr[vi], gu = gr[vi];
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
        const float inv = 1.0f / sqrtf(ss / static_cast<float>(hid) + c.rms_eps);
        const float z = dot * inv + (bias ? to_f(bias[h]) : 0.f);
        const float a = z * c.alpha_scale - da.offset[b * da.offset_bstride + h];
        if (layer_mode)
          for (int hh = 0; hh < c.Hkv; ++hh) alpha[b * c.Hkv + hh] = a;
        else
          alpha[b * c.Hkv + h] = a;
      }
    }
    __syncthreads();
  }
  DMS_TRACE_MARK(1, 1);
  // Phase 1: slots and page grants
  for (int i0 = 0; i0 < BH; i0 += bd) {
    const int i = i0 + tid;
    int need = 0, slot = -1, cnt = 0, have = 0;
    bool reuse = false, evict = false;
    const long li = lbase + i;
    int t = 0;
    if (i < BH) {
      const int b = i / c.Hkv, h = i % c.Hkv;
      t = c.pos[layer * c.B + b];  // position of the new token
      const int hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
      evict = !c.disable && alpha[b * c.Hkv + hs] > 0.0f;
      const int ringv = t >= w ? c.ring[li * w + t % w] : 0;
      reuse = t >= w && (static_cast<unsigned>(ringv) & RING_EVICT);
      cnt = c.count[li];
      have = c.npages[li];
      if (reuse) {
        slot = ringv & RING_SLOT_MASK;
      } else if (cnt >= c.cap) {
        set_status(c.ctrl, DMS_ST_CAPACITY);
      } else {
        slot = cnt;
        need = (cnt % P == 0 && cnt / P >= have) ? 1 : 0;
      }
    }
    int tot;
    const int off = block_exclusive_scan(need, tmp, &tot);
    if (i < BH) {
      int id = -1;
      bool ok = slot >= 0;
      if (ok && need) {
        id = next + off;
        if (id < c.pool_pages && have < c.maxp) {
          c.page_table[li * c.maxp + have] = id;
          c.npages[li] = have + 1;
        } else {
          set_status(c.ctrl, DMS_ST_POOL_EXHAUSTED);
          ok = false;
        }
      }
      if (ok) {
        const int newcnt = reuse ? cnt : cnt + 1;
        if (!reuse) c.count[li] = newcnt;
        const int p = slot / P;
        s_slot[i] = slot;
        s_id[i] = need ? id : c.page_table[li * c.maxp + p];
        s_rows[i] = min(P, newcnt - p * P);
        c.slot_pos[li * c.cap + slot] = t;
        c.ring[li * w + t % w] = slot | (evict ? static_cast<int>(RING_EVICT) : 0);
      } else {
        s_slot[i] = -1;
      }
    }
    next += tot;
  }
  if (tid == 0) c.ctrl[CTRL_NEXT_PAGE] = min(next, c.pool_pages);
  __syncthreads();  // every head has read its position
  for (int b = tid; b < c.B; b += bd) c.pos[layer * c.B + b] += 1;

  DMS_TRACE_MARK(1, 2);
  // Phase 2: K/V rows, one warp per head
  const int D = c.D;
  for (int i = wid; i < BH; i += nwarp) {
    const int slot = s_slot[i];
    if (slot < 0) continue;
    const int id = s_id[i];
    const long dst_row = static_cast<long>(id) * P + slot % P;
    const TA* ksrc = k + static_cast<long>(i) * D;
    const TA* vsrc = v + static_cast<long>(i) * D;
    if (!FP8) {
      const int cpr = D * static_cast<int>(sizeof(TA)) / 16;
      if (lane < cpr) {
        reinterpret_cast<uint4*>(static_cast<TA*>(c.k_pool) + dst_row * D)[lane] =
            reinterpret_cast<const uint4*>(ksrc)[lane];
        reinterpret_cast<uint4*>(static_cast<TA*>(c.v_pool) + dst_row * D)[lane] =
            reinterpret_cast<const uint4*>(vsrc)[lane];
      }
    } else {
      const int rows = s_rows[i];
      for (int which = 0; which < 2; ++which) {
        const TA* x = which ? vsrc : ksrc;
        float* scale_p = (which ? c.v_scale : c.k_scale) + id;
        uint8_t* page = static_cast<uint8_t*>(which ? c.v_pool : c.k_pool) + static_cast<long>(id) * P * D;
        float xv[4];
        float amax = 0.f;
        for (int e = 0; e < D / 32; ++e) {
          xv[e] = to_f(x[lane + 32 * e]);
          amax = fmaxf(amax, fabsf(xv[e]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s_new = __fdiv_rn(amax, 448.0f);
        const float s_old = *scale_p;
        float scale = s_old;
        if (s_new > s_old) {
          // re-encode the page's rows at the larger scale from their decoded values
          for (int idx = lane; idx < rows * D; idx += 32) {
            const float dq = __fmul_rn(fp8_decode(page[idx]), s_old);
            page[idx] = fp8_encode(__fdiv_rn(dq, s_new));
          }
          scale = s_new;
          __syncwarp();
          if (lane == 0) *scale_p = s_new;
        }
        for (int e = 0; e < D / 32; ++e)
          page[static_cast<long>(slot % P) * D + lane + 32 * e] = scale > 0.f ? fp8_encode(__fdiv_rn(xv[e], scale)) : 0;
      }
    }
  }

  // Phase 3: slot plan of the next append of every head (read by the fused
  // decode kernel).
  __syncthreads();
  for (int i = tid; i < BH; i += bd) {
    const int b = i / c.Hkv;
    c.plan[lbase + i] = next_plan(c, lbase + i, c.pos[layer * c.B + b]);
  }
  DMS_TRACE_MARK(1, 3);
}

template <typename TA, bool FP8>
static cudaError_t launch_append_t(const CacheView& c, int layer, const void* k, const void* v, float* alpha,
                                   const DecideArgs* da, int threads, size_t smem, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(k_decode_append<TA, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  DecideArgs none{};
  k_decode_append<TA, FP8><<<1, threads, smem, s>>>(c, layer, static_cast<const TA*>(k), static_cast<const TA*>(v),
                                                    alpha, da ? *da : none, da ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_decode_append(const CacheView& c, int layer, const void* k, const void* v, float* alpha,
                                 const DecideArgs* fused_decide, int num_sms, cudaStream_t s) {
  const int BH = c.B * c.Hkv;
  (void)num_sms;
  const int threads = min(1024, max(256, (BH + 31) / 32 * 32));
  const size_t smem = static_cast<size_t>(BH) * 3 * sizeof(int);
  if (c.kv_dtype == DMS_FP8_E4M3)
    return launch_append_t<__nv_bfloat16, true>(c, layer, k, v, alpha, fused_decide, threads, smem, s);
  if (c.kv_dtype == DMS_BF16)
    return launch_append_t<__nv_bfloat16, false>(c, layer, k, v, alpha, fused_decide, threads, smem, s);
  return launch_append_t<float, false>(c, layer, k, v, alpha, fused_decide, threads, smem, s);
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
// bf16 / FP8 split-K decode attention ([FastDMS], attention scoring: split-K
// grouped compact decode attention over variable-length per-head live spans).
//
// Every CTA derives the same work partition from the heads' retained counts
// and walks its items (chunks of one head's slots inside one page) in grid
// stride.  Sub-tiles of 64 slots are staged by TMA (16-row boxes, no
// multicast) into a ring of shared-memory stages; 4 warps take 16 slots each
// and run QK^T and PV on mma.sync with the g query heads of the KV head as the
// M dimension (padded to 16), so every K/V byte is read once per step.  Each
// item leaves an unnormalised partial (acc, running max, running sum, log2
// domain); the CTA that finishes a head's last item (per-head arrival
// counter) merges the head's partials and writes its output rows.
// bf16 pages arrive with the 128-byte swizzle; FP8 pages arrive unswizzled and
// are widened to bf16 codes (exact) in shared memory, their page scale applied
// to the scores (K) and to the partial (V).
//
// FUSED (bf16 pages): the whole decode step in one launch.  The attention runs
// over the slots as they were before this step's append, with the slot about
// to be reused masked out and the new token's key/value taken from the input
// as one more key of the head's first item -- the same visible set as after
// the append.  The CTA that merges a head then appends that head's token (the
// slot plan was fixed by the previous step), and the last CTA of the grid
// updates the counts, page counter and positions and plans the next append.
// Page ids are granted in (b, h) row-major order, as in the one-CTA append.
// ---------------------------------------------------------------------------
struct FusedArgs {
  const __nv_bfloat16* k_new;  // [B, Hkv, D]
  const __nv_bfloat16* v_new;  // [B, Hkv, D]
  float* alpha;                // [B, Hkv] decision logits (written here when decide is fused)
  DecideArgs da;
  int fuse_decide;
};

// Adapter decision logit of the new token of sequence b for head `src`, by one
// CTA (all loads of a thread issued before use).  Returns the value in thread 0.
template <int HID_VEC_PER_THREAD>
__device__ __forceinline__ float decide_cta(const CacheView& c, const DecideArgs& a, int b, int src, float* red) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int hid = c.hidden, nvec = hid / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.hidden) + static_cast<long>(b) * hid);
  const uint4* wr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.W) + static_cast<long>(src) * hid);
  const uint4* gr = reinterpret_cast<const uint4*>(a.gamma);
  float ss = 0.f, dot = 0.f;
  for (int v0 = 0; v0 < nvec; v0 += kThreads * HID_VEC_PER_THREAD) {
    uint4 xu[HID_VEC_PER_THREAD], wu[HID_VEC_PER_THREAD], gu[HID_VEC_PER_THREAD];
#pragma unroll
    for (int u = 0; u < HID_VEC_PER_THREAD; ++u) {
      const int vi = v0 + u * kThreads + tid;
      const bool ok = vi < nvec;
      xu[u] = ok ? xr[vi] : make_uint4(0, 0, 0, 0);
      wu[u] = ok ? wr[vi] : make_uint4(0, 0, 0, 0);
      gu[u] = ok ? gr[vi] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < HID_VEC_PER_THREAD; ++u) {
      float x[8], wv[8], gv[8];
      unpack16(xu[u], x, static_cast<const __nv_bfloat16*>(nullptr));
      unpack16(wu[u], wv, static_cast<const __nv_bfloat16*>(nullptr));
      unpack16(gu[u], gv, static_cast<const __nv_bfloat16*>(nullptr));
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ss = fmaf(x[e], x[e], ss);
        dot = fmaf(wv[e] * gv[e], x[e], dot);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
  }
  __syncthreads();
  if (lane == 0) {
    red[wid] = ss;
    red[4 + wid] = dot;
  }
  __syncthreads();
  float alpha = 0.f;
  if (tid == 0) {
    const float s2 = red[0] + red[1] + red[2] + red[3];
    const float d2 = red[4] + red[5] + red[6] + red[7];
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(a.bias);
    const float inv = 1.0f / sqrtf(s2 / static_cast<float>(hid) + c.rms_eps);
    const float z = d2 * inv + (bias ? __bfloat162float(bias[src]) : 0.f);
    alpha = z * c.alpha_scale - a.offset[b * a.offset_bstride + src];
  }
  return alpha;
}

// Number of heads before `bh` of this layer whose planned append needs a new page.
__device__ __forceinline__ int new_page_rank(const int2* plan, int bh, int* red) {
  int n = 0;
  for (int i = threadIdx.x; i < bh; i += kThreads) n += (plan[i].y & 2) ? 1 : 0;
  int tot;
  block_exclusive_scan(n, red, &tot);
  return tot;
}

template <int D, bool FP8, bool FUSED>
__global__ void __launch_bounds__(kThreads) k_decode_attn(CacheView c, int layer, const __nv_bfloat16* q,
                                                         __nv_bfloat16* o, int target_items, FusedArgs fa,
                                                         const __grid_constant__ CUtensorMap kmap,
                                                         const __grid_constant__ CUtensorMap vmap) {
  using S = DecodeSmem<D, FP8>;
  constexpr int KS = D / 16, NT = D / 8, MLD = D + 2;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sbase =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* stage_buf = sbase;                         // kStages * STAGE
  unsigned char* conv_buf = sbase + kStages * S::STAGE;     // FP8: widened K, V
  float* merge = reinterpret_cast<float*>(conv_buf + S::CONV);  // [5 sources][g rows][D + 2]
  const int g = c.Hq / c.Hkv;
  const int BH = c.B * c.Hkv;
  int* s_off = reinterpret_cast<int*>(merge + 5 * g * MLD);  // [BH + 1] first work item of each head
  int* s_cnt = s_off + BH + 1;                               // [BH] retained slots of each head
  float* wbuf = reinterpret_cast<float*>(s_cnt + BH);        // [2 * kCombineChunk + 32] combine staging
  __shared__ uint64_t full_bar[kStages];
  __shared__ StageMeta meta[kStages];
  __shared__ int s_abort, s_last, s_have, s_next_page;
  __shared__ int s_red[32][4];
  __shared__ float s_fred[8];

  const int tid = threadIdx.x;
  const long lbase = static_cast<long>(layer) * BH;
  DMS_TRACE_MARK(0, 0);
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&full_bar[i], 1);
    fence_mbar_init();
    s_abort = 0;
    if (FUSED) s_next_page = c.ctrl[CTRL_NEXT_PAGE];
  }
  const int C = decode_partition(c.count + lbase, BH, c.P, target_items, s_cnt, s_off, s_red);
  const int nitems = s_off[BH];
  DMS_TRACE_MARK(0, 1);

  // producer iterator (thread 0 only)
  int p_item = blockIdx.x, p_sub = 0, p_bh = 0;
  auto produce = [&](int stage) -> bool {
    while (p_item < nitems) {
      while (s_off[p_bh + 1] <= p_item) ++p_bh;  // items are visited in increasing order
      const int s0 = (p_item - s_off[p_bh]) * C;
      const int len = min(s_cnt[p_bh], s0 + C) - s0;
      if (p_sub < len) {
        const long lbh = lbase + p_bh;
        const int slot0 = s0 + p_sub;
        const int page = c.page_table[lbh * c.maxp + slot0 / c.P];
        const int rows = min(kSub, len - p_sub);
        StageMeta& m = meta[stage];
        m.item = p_item;
        m.bh = p_bh;
        m.s0 = s0;
        m.sub = p_sub;
        m.rows = rows;
        m.page = page;
        m.last = (p_sub + kSub >= len) ? 1 : 0;
        const int nbox = (rows + 15) / 16;
        const int row0 = page * c.P + slot0 % c.P;
        unsigned char* dst = stage_buf + stage * S::STAGE;
        const uint32_t bytes = static_cast<uint32_t>(nbox * 16 * (FP8 ? D : 128) * (FP8 ? 1 : S::HALVES) * 2);
        mbar_expect_tx(&full_bar[stage], bytes);
        for (int bx = 0; bx < nbox; ++bx) {
          if (FP8) {
            tma_load_2d(dst + bx * 16 * D, &kmap, 0, row0 + bx * 16, &full_bar[stage]);
            tma_load_2d(dst + S::TILE_RAW + bx * 16 * D, &vmap, 0, row0 + bx * 16, &full_bar[stage]);
          } else {
            for (int hf = 0; hf < S::HALVES; ++hf) {
              tma_load_2d(dst + hf * kSub * 128 + bx * 16 * 128, &kmap, hf * 64, row0 + bx * 16, &full_bar[stage]);
              tma_load_2d(dst + S::TILE_RAW + hf * kSub * 128 + bx * 16 * 128, &vmap, hf * 64, row0 + bx * 16,
                          &full_bar[stage]);
            }
          }
        }
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

  // per-item consumer state
  uint32_t qa[KS][4];
  float acc[NT][4];
  float mrow[2], lrow[2];
  int cur_item = -1, masked_slot = -1;
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
    const long li = lbase + bh;
    if (n == 0) DMS_TRACE_MARK(0, 2);
    const unsigned char* kt;
    const unsigned char* vt;
    if (FP8) {
      // widen FP8 codes to bf16 in the swizzled layout
      const uint8_t* raw = stage_buf + stage * S::STAGE;
      for (int idx = tid; idx < 2 * kSub * (D / 16); idx += kThreads) {
        const int which = idx / (kSub * (D / 16));
        const int rem = idx % (kSub * (D / 16));
        const int r = rem / (D / 16), ch = rem % (D / 16);  // 16 codes
        const uint4 u = *reinterpret_cast<const uint4*>(raw + which * S::TILE_RAW + r * D + ch * 16);
        const uint8_t* cb = reinterpret_cast<const uint8_t*>(&u);
        uint32_t wds[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) wds[e] = pack_bf16(fp8_decode(cb[2 * e]), fp8_decode(cb[2 * e + 1]));
        unsigned char* dstt = conv_buf + which * S::TILE_BF16;
        for (int hc = 0; hc < 2; ++hc) {
          const int chunk = 2 * ch + hc;
          *reinterpret_cast<uint4*>(dstt + (chunk / 8) * kSub * 128 + sw128(r, chunk % 8)) =
              make_uint4(wds[4 * hc], wds[4 * hc + 1], wds[4 * hc + 2], wds[4 * hc + 3]);
        }
      }
      __syncthreads();
      kt = conv_buf;
      vt = conv_buf + S::TILE_BF16;
    } else {
      kt = stage_buf + stage * S::STAGE;
      vt = kt + S::TILE_RAW;
    }

    const bool first_of_head = FUSED && m.s0 == 0;
    if (m.item != cur_item) {
      cur_item = m.item;
      load_q_frags<D>(q + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D, g, qa);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      mrow[0] = mrow[1] = -INFINITY;
      lrow[0] = lrow[1] = 0.f;
      if (FUSED) {
        const int2 pl = c.plan[li];
        masked_slot = (pl.y & 1) ? pl.x : -1;  // the slot this step's token reuses
        if (first_of_head && fa.fuse_decide) {
          // decision logit of the new token (layer granularity: head 0's)
          const int src = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
          const float a = decide_cta<4>(c, fa.da, b, src, s_fred);
          if (tid == 0) fa.alpha[b * c.Hkv + h] = a;
        }
      }
    }

    const int warp = tid >> 5;
    if (warp * 16 < m.rows) {
      const float kscale = FP8 ? c.k_scale[m.page] : 1.0f;
      const int masked = masked_slot - (m.s0 + m.sub);
      warp_tile<D>(kt, vt, m.rows, masked, kscale * sl2, qa, acc, mrow, lrow);
    }
    __syncthreads();  // every warp is done with this stage (and with conv_buf)
    if (tid == 0 && produce(stage)) ++produced;

    if (m.last) {
      if (n == 0) DMS_TRACE_MARK(0, 3);
      warp_state_to_smem<D>(merge, warp, g, acc, mrow, lrow);
      int nsrc = 4;
      if (first_of_head) {
        // the new token as a fifth source: score q_r . k_new, weight 1, value v_new
        const __nv_bfloat16* kn = fa.k_new + static_cast<long>(bh) * D;
        const __nv_bfloat16* vn = fa.v_new + static_cast<long>(bh) * D;
        const __nv_bfloat16* qb = q + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D;
        const int lane = tid & 31;
        for (int r = warp; r < g; r += 4) {
          float sdot = 0.f;
          for (int d = lane; d < D; d += 32)
            sdot = fmaf(__bfloat162float(qb[static_cast<long>(r) * D + d]), __bfloat162float(kn[d]), sdot);
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o2);
          if (lane == 0) {
            merge[(4 * g + r) * MLD + D] = sdot * sl2;
            merge[(4 * g + r) * MLD + D + 1] = 1.0f;
          }
        }
        for (int idx = tid; idx < g * D; idx += kThreads)
          merge[(4 * g + idx / D) * MLD + idx % D] = __bfloat162float(vn[idx % D]);
        nsrc = 5;
      }
      __syncthreads();
      const float vscale = FP8 ? c.v_scale[m.page] : 1.0f;
      merge_to_partial<D>(merge, nsrc, g, vscale, c.part_acc, c.part_ml, m.item);
      cur_item = -1;
      // the last CTA to finish one of this head's items merges the head
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        const int nh = s_off[bh + 1] - s_off[bh];
        s_last = (atomicAdd(&c.head_done[bh], 1) == nh - 1) ? 1 : 0;
      }
      __syncthreads();
      DMS_TRACE_MARK(0, 4);
      if (s_last) {
        __threadfence();
        combine_head<D>(c.part_acc, c.part_ml, g, s_off[bh], s_off[bh + 1],
                        o + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D, wbuf);
        if (FUSED) {
          // append of this head's token at the planned slot
          const int2 pl = c.plan[li];
          int id = -1;
          bool ok = !(pl.y & 4);
          if (pl.y & 2) {
            const int rank = new_page_rank(c.plan + lbase, bh, &s_red[0][0]);
            id = s_next_page + rank;
            if (id >= c.pool_pages || c.npages[li] >= c.maxp) ok = false;
          } else if (ok) {
            id = c.page_table[li * c.maxp + pl.x / c.P];
          }
          if (ok) {
            const int t = c.pos[layer * c.B + b];
            if ((pl.y & 2) && tid == 0) c.page_table[li * c.maxp + c.npages[li]] = id;
            const long row = static_cast<long>(id) * c.P + pl.x % c.P;
            if (tid < D / 8) {
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.k_pool) + row * D)[tid] =
                  reinterpret_cast<const uint4*>(fa.k_new + static_cast<long>(bh) * D)[tid];
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.v_pool) + row * D)[tid] =
                  reinterpret_cast<const uint4*>(fa.v_new + static_cast<long>(bh) * D)[tid];
            }
            if (tid == 0) {
              const int hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
              const bool evict = !c.disable && __ldcg(&fa.alpha[b * c.Hkv + hs]) > 0.0f;
              c.slot_pos[li * c.cap + pl.x] = t;
              c.ring[li * c.w + t % c.w] = pl.x | (evict ? static_cast<int>(RING_EVICT) : 0);
            }
          } else if (tid == 0) {
            set_status(c.ctrl, (pl.y & 4) ? DMS_ST_CAPACITY : DMS_ST_POOL_EXHAUSTED);
          }
        }
        if (tid == 0) c.head_done[bh] = 0;
        DMS_TRACE_MARK(0, 5);
      }
    }
  }

  if (FUSED) {
    // the last CTA of the grid updates the per-head counts, the page counter
    // and the positions, then plans the next append of every head
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&c.ctrl[CTRL_GRID_DONE], 1) == static_cast<int>(gridDim.x) - 1) ? 1 : 0;
    __syncthreads();
    if (s_last) {
      __threadfence();
      int next = s_next_page;
      for (int i0 = 0; i0 < BH; i0 += kThreads) {
        const int i = i0 + tid;
        const int2 pl = i < BH ? __ldcg(&c.plan[lbase + i]) : make_int2(0, 0);
        const int need = (i < BH && (pl.y & 2)) ? 1 : 0;
        int tot;
        const int off = block_exclusive_scan(need, &s_red[0][0], &tot);
        if (i < BH) {
          const long li = lbase + i;
          const bool granted = need && next + off < c.pool_pages && c.npages[li] < c.maxp;
          const bool dropped = (pl.y & 4) || (need && !granted);
          if (!dropped && !(pl.y & 1)) c.count[li] += 1;
          if (granted) c.npages[li] += 1;
        }
        next += tot;
      }
      if (tid == 0) c.ctrl[CTRL_NEXT_PAGE] = min(next, c.pool_pages);
      for (int b = tid; b < c.B; b += kThreads) c.pos[layer * c.B + b] += 1;
      __syncthreads();
      for (int i = tid; i < BH; i += kThreads)
        c.plan[lbase + i] = next_plan(c, lbase + i, c.pos[layer * c.B + i / c.Hkv]);
      if (tid == 0) c.ctrl[CTRL_GRID_DONE] = 0;
    }
  }
  DMS_TRACE_MARK(0, 6);
}

template <int D, bool FP8, bool FUSED>
static cudaError_t launch_attn(const CacheView& c, int layer, const void* q, void* o, const FusedArgs& fa,
                               const CUtensorMap* kmap, const CUtensorMap* vmap, int num_sms, cudaStream_t s) {
  using S = DecodeSmem<D, FP8>;
  const int g = c.Hq / c.Hkv;
  const size_t smem = 1024 + kStages * S::STAGE + S::CONV + 5 * g * (D + 2) * sizeof(float) +
                      (2 * static_cast<size_t>(c.B) * c.Hkv + 1) * sizeof(int) + (2 * kCombineChunk + 32) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_decode_attn<D, FP8, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = 2 * num_sms;
  k_decode_attn<D, FP8, FUSED><<<grid, kThreads, smem, s>>>(c, layer, static_cast<const __nv_bfloat16*>(q),
                                                            static_cast<__nv_bfloat16*>(o), 2 * min(num_sms, 160), fa,
                                                            *kmap, *vmap);
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
  const FusedArgs none{};
  if (c.kv_dtype == DMS_FP8_E4M3)
    return c.D == 64 ? launch_attn<64, true, false>(c, layer, q, o, none, kmap, vmap, num_sms, s)
                     : launch_attn<128, true, false>(c, layer, q, o, none, kmap, vmap, num_sms, s);
  return c.D == 64 ? launch_attn<64, false, false>(c, layer, q, o, none, kmap, vmap, num_sms, s)
                   : launch_attn<128, false, false>(c, layer, q, o, none, kmap, vmap, num_sms, s);
}

cudaError_t launch_decode_fused(const CacheView& c, int layer, const void* q, const void* k, const void* v, void* o,
                                float* alpha, const DecideArgs* fused_decide, const CUtensorMap* kmap,
                                const CUtensorMap* vmap, int num_sms, cudaStream_t s) {
  if (c.kv_dtype != DMS_BF16 || !kmap || !vmap) return cudaErrorInvalidValue;
  FusedArgs fa{};
  fa.k_new = static_cast<const __nv_bfloat16*>(k);
  fa.v_new = static_cast<const __nv_bfloat16*>(v);
  fa.alpha = alpha;
  if (fused_decide) {
    fa.da = *fused_decide;
    fa.fuse_decide = 1;
  }
  return c.D == 64 ? launch_attn<64, false, true>(c, layer, q, o, fa, kmap, vmap, num_sms, s)
                   : launch_attn<128, false, true>(c, layer, q, o, fa, kmap, vmap, num_sms, s);
}

}  // namespace dms

#ifdef DMS_TRACE
// Copy the phase timeline to the host (tracing builds only).
extern "C" __attribute__((visibility("default"))) int dms_debug_trace_read(void* host, size_t bytes) {
  const size_t n = sizeof(dms::g_dms_trace) < bytes ? sizeof(dms::g_dms_trace) : bytes;
  return cudaMemcpyFromSymbol(host, dms::g_dms_trace, n) == cudaSuccess ? 0 : -3;
}
extern "C" __attribute__((visibility("default"))) int dms_debug_trace_clear() {
  static unsigned long long zeros[2 * dms::kTraceCtas * dms::kTraceSlots];
  return cudaMemcpyToSymbol(dms::g_dms_trace, zeros, sizeof(zeros)) == cudaSuccess ? 0 : -3;
}
#endif
