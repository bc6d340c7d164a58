// Decode step: append with delayed eviction, then split-K grouped attention
// over each head's compact retained slots.
#include "dms_internal.cuh"

namespace dms {

// ---------------------------------------------------------------------------
// Append of token t for every (b, h) of one layer, in one CTA so that page
// grants follow (b, h) row-major order without inter-CTA ordering:
//   if t >= w and the token t - w (ring[t % w]) was marked for eviction, the new
//   token overwrites its slot in place; else it takes slot count++, and a page
//   is granted from the ascending counter when that slot starts a page
//   ([DMS-Qwen3], inference mode with the paged KV cache; [FastDMS], decode
//   kernel: per-step keep/evict, sliding retention window, compact append).
// The same CTA then writes the K/V rows (FP8: re-encodes the page when the new
// row raises its scale) and builds the work list of the attention kernel.
// ---------------------------------------------------------------------------
template <typename TA, bool FP8>
__global__ void __launch_bounds__(1024) k_decode_append(CacheView c, int layer, const TA* k, const TA* v,
                                                       const float* alpha, int target_items) {
  extern __shared__ int sh[];
  __shared__ int tmp[32];
  const int BH = c.B * c.Hkv;
  int* s_slot = sh;          // slot written by head i (-1: dropped)
  int* s_id = sh + BH;       // page id holding that slot
  int* s_rows = sh + 2 * BH; // rows in use in that page after the append
  const long lbase = static_cast<long>(layer) * BH;
  const int tid = threadIdx.x, bd = blockDim.x, w = c.w, P = c.P;
  int next = c.ctrl[CTRL_NEXT_PAGE];

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

  // Phase 2: K/V rows, one warp per head
  const int lane = tid & 31, wid = tid >> 5, nwarp = bd >> 5;
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

  // Phase 3: work list of the split-K attention.  Chunk C (a power-of-two
  // divisor of P, >= 16) is the largest giving at least `target_items` items.
  int C = P;
  while (true) {
    int part = 0;
    for (int i = tid; i < BH; i += bd) part += (c.count[lbase + i] + C - 1) / C;
    int tot;
    block_exclusive_scan(part, tmp, &tot);
    if (tot >= target_items || (C / 2) % 16 != 0 || (P % (C / 2)) != 0) break;
    C /= 2;
  }
  int base = 0;
  for (int i0 = 0; i0 < BH; i0 += bd) {
    const int i = i0 + tid;
    const int cnt = i < BH ? c.count[lbase + i] : 0;
    const int n = (cnt + C - 1) / C;
    int tot;
    const int off = block_exclusive_scan(n, tmp, &tot);
    if (i < BH) {
      c.item_off[i] = base + off;
      for (int j = 0; j < n; ++j) {
        const int it = base + off + j;
        if (it < c.items_cap)
          c.items[it] = make_int4(i, j * C, min(cnt, (j + 1) * C), 0);
        else
          set_status(c.ctrl, DMS_ST_CAPACITY);
      }
    }
    base += tot;
  }
  if (tid == 0) {
    c.item_off[BH] = min(base, c.items_cap);
    c.ctrl[CTRL_NITEMS] = min(base, c.items_cap);
    c.ctrl[CTRL_CHUNK] = C;
  }
}

cudaError_t launch_decode_append(const CacheView& c, int layer, const void* k, const void* v,
                                 const float* alpha, int num_sms, cudaStream_t s) {
  const int BH = c.B * c.Hkv;
  const int threads = min(1024, max(128, (BH + 31) / 32 * 32));
  const size_t smem = static_cast<size_t>(BH) * 3 * sizeof(int);
  const int target = 2 * min(num_sms, 160);
  cudaError_t e;
  if (c.kv_dtype == DMS_FP8_E4M3) {
    e = cudaFuncSetAttribute(k_decode_append<__nv_bfloat16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_decode_append<__nv_bfloat16, true><<<1, threads, smem, s>>>(c, layer, static_cast<const __nv_bfloat16*>(k),
                                                                  static_cast<const __nv_bfloat16*>(v), alpha, target);
  } else if (c.kv_dtype == DMS_BF16) {
    e = cudaFuncSetAttribute(k_decode_append<__nv_bfloat16, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_decode_append<__nv_bfloat16, false><<<1, threads, smem, s>>>(
        c, layer, static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), alpha, target);
  } else {
    e = cudaFuncSetAttribute(k_decode_append<float, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_decode_append<float, false><<<1, threads, smem, s>>>(c, layer, static_cast<const float*>(k),
                                                           static_cast<const float*>(v), alpha, target);
  }
  return cudaGetLastError();
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
// bf16 / FP8 split-K decode attention.
//
// Persistent CTAs walk the work list; each item is a chunk [s0, s1) of one
// head's slots inside one page.  Sub-tiles of 64 slots are staged by TMA
// (16-row boxes, no multicast) into a ring of shared-memory stages; 4 warps
// take 16 slots each and run QK^T and PV on mma.sync with the g query heads of
// the KV head as the M dimension (padded to 16), so every K/V byte is read
// once per step.  Each item leaves an unnormalised partial (acc, running max,
// running sum, log2 domain) for the combine kernel.
// bf16 pages arrive with the 128-byte swizzle; FP8 pages arrive unswizzled and
// are widened to bf16 codes (exact) in shared memory, their page scale applied
// to the scores (K) and to the partial (V).
// ---------------------------------------------------------------------------
constexpr int kSub = 64;     // slots per sub-tile
constexpr int kStages = 3;

template <int D, bool FP8>
struct DecodeSmem {
  static constexpr int HALVES = D / 64;                    // 128-byte column halves of a bf16 row
  static constexpr int TILE_BF16 = kSub * D * 2;           // bytes of one bf16 K (or V) sub-tile
  static constexpr int TILE_RAW = FP8 ? kSub * D : TILE_BF16;
  static constexpr int STAGE = 2 * TILE_RAW;               // K then V, as loaded
  static constexpr int CONV = FP8 ? 2 * TILE_BF16 : 0;     // widened bf16 K and V (FP8 only)
};

struct StageMeta {
  int item;    // work item index
  int sub;     // first slot of the sub-tile, relative to the item start
  int rows;    // valid slots in the sub-tile
  int page;    // page id
  int last;    // 1 if this is the item's last sub-tile
};

__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  // byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled tile
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int D, bool FP8>
__global__ void __launch_bounds__(128) k_decode_attn(CacheView c, int layer, const __nv_bfloat16* q,
                                                    const __grid_constant__ CUtensorMap kmap,
                                                    const __grid_constant__ CUtensorMap vmap) {
  using S = DecodeSmem<D, FP8>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sbase = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* stage_buf = sbase;                                  // kStages * STAGE
  unsigned char* conv_buf = sbase + kStages * S::STAGE;              // FP8: widened K, V
  float* merge = reinterpret_cast<float*>(conv_buf + S::CONV);       // [4 warps][g rows][D + 2]
  __shared__ uint64_t full_bar[kStages];
  __shared__ StageMeta meta[kStages];
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nitems = c.ctrl[CTRL_NITEMS];
  const int g = c.Hq / c.Hkv;
  const long lbase = static_cast<long>(layer) * c.B * c.Hkv;
  constexpr int KS = D / 16;
  constexpr int NT = D / 8;
  constexpr int MLD = D + 2;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&full_bar[i], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();

  // producer iterator (thread 0 only)
  int p_item = blockIdx.x, p_sub = 0;
  auto produce = [&](int stage) -> bool {
    while (p_item < nitems) {
      const int4 it = c.items[p_item];
      const int len = it.z - it.y;
      if (p_sub < len) {
        const long lbh = lbase + it.x;
        const int slot0 = it.y + p_sub;
        const int page = c.page_table[lbh * c.maxp + slot0 / c.P];
        const int rows = min(kSub, len - p_sub);
        StageMeta& m = meta[stage];
        m.item = p_item;
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
  if (tid == 0) {
    for (int st = 0; st < kStages; ++st)
      if (produce(st)) ++produced;
  }

  // per-item consumer state
  uint32_t qa[KS][4];
  float acc[NT][4];
  float mrow[2], lrow[2];
  int cur_item = -1;
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  const int ra = lane >> 2, rb = ra + 8;  // query-head rows of this thread

  for (int n = 0;; ++n) {
    // Is there an n-th sub-tile for this CTA?  Recompute the consumer iterator.
    // (All threads follow the same deterministic sequence as the producer.)
    __syncthreads();
    if (s_abort) break;
    const int stage = n % kStages;
    // the producer has filled `produced` sub-tiles so far; stop when none is pending
    __shared__ int s_have;
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
    const int4 it = c.items[m.item];
    const int bh = it.x, b = bh / c.Hkv, h = bh % c.Hkv;
    const unsigned char* kt;
    const unsigned char* vt;
    if (FP8) {
      // widen FP8 codes to bf16 in the swizzled layout
      const uint8_t* raw = stage_buf + stage * S::STAGE;
      for (int idx = tid; idx < 2 * kSub * (D / 16); idx += 128) {
        const int which = idx / (kSub * (D / 16));
        const int rem = idx % (kSub * (D / 16));
        const int r = rem / (D / 16), ch = rem % (D / 16);  // 16 codes
        const uint4 u = *reinterpret_cast<const uint4*>(raw + which * S::TILE_RAW + r * D + ch * 16);
        const uint8_t* cb = reinterpret_cast<const uint8_t*>(&u);
        uint32_t wds[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) wds[e] = pack_bf16(fp8_decode(cb[2 * e]), fp8_decode(cb[2 * e + 1]));
        unsigned char* dstt = conv_buf + which * S::TILE_BF16;
        // bf16 row of D elements: 16-byte chunks 2*ch and 2*ch+1, column half = chunk / 8
        for (int hc = 0; hc < 2; ++hc) {
          const int chunk = 2 * ch + hc;
          const int hf = chunk / 8, cc = chunk % 8;
          *reinterpret_cast<uint4*>(dstt + hf * kSub * 128 + sw128(r, cc)) =
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

    if (m.item != cur_item) {
      cur_item = m.item;
      // Q fragments of the g query heads (rows >= g are zero)
      const __nv_bfloat16* qb = q + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int col = ks * 16 + 2 * (lane & 3);
        auto ld = [&](int r, int cc) -> uint32_t {
          return r < g ? *reinterpret_cast<const uint32_t*>(qb + static_cast<long>(r) * D + cc) : 0u;
        };
        qa[ks][0] = ld(ra, col);
        qa[ks][1] = ld(rb, col);
        qa[ks][2] = ld(ra, col + 8);
        qa[ks][3] = ld(rb, col + 8);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      mrow[0] = mrow[1] = -INFINITY;
      lrow[0] = lrow[1] = 0.f;
    }

    if (warp * 16 < m.rows) {
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int n_row = warp * 16 + (mi >> 1) * 8 + rr;
        const int chunk = 2 * ks + (mi & 1);
        const uint32_t addr = smem_u32(kt + (chunk / 8) * kSub * 128 + sw128(n_row, chunk % 8));
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(b0, b1, b2, b3, addr);
        uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
        mma_bf16_16816(s[0], qa[ks], bb0);
        mma_bf16_16816(s[1], qa[ks], bb1);
      }
      const float kscale = FP8 ? c.k_scale[m.page] : 1.0f;
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = warp * 16 + nt * 8 + 2 * (lane & 3) + (e & 1);
          const float x = key < m.rows ? s[nt][e] * kscale * sl2 : -INFINITY;
          s[nt][e] = x;
          mx[e >> 1] = fmaxf(mx[e >> 1], x);
        }
      float corr[2], mu[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        const float mn = fmaxf(mrow[r], mx[r]);
        mu[r] = mn == -INFINITY ? 0.f : mn;
        corr[r] = exp2f(mrow[r] - mu[r]);
        mrow[r] = mn;
      }
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p = exp2f(s[nt][e] - mu[e >> 1]);
          s[nt][e] = p;
          rs[e >> 1] += p;
        }
      lrow[0] = lrow[0] * corr[0] + rs[0];
      lrow[1] = lrow[1] * corr[1] + rs[1];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[nt][0] *= corr[0];
        acc[nt][1] *= corr[0];
        acc[nt][2] *= corr[1];
        acc[nt][3] *= corr[1];
      }
      uint32_t pa[4];
      pa[0] = pack_bf16(s[0][0], s[0][1]);
      pa[1] = pack_bf16(s[0][2], s[0][3]);
      pa[2] = pack_bf16(s[1][0], s[1][1]);
      pa[3] = pack_bf16(s[1][2], s[1][3]);
#pragma unroll
      for (int dp = 0; dp < NT / 2; ++dp) {
        const int n_row = warp * 16 + (mi & 1) * 8 + rr;
        const int chunk = 2 * dp + (mi >> 1);
        const uint32_t addr = smem_u32(vt + (chunk / 8) * kSub * 128 + sw128(n_row, chunk % 8));
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(b0, b1, b2, b3, addr);
        uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
        mma_bf16_16816(acc[2 * dp], pa, bb0);
        mma_bf16_16816(acc[2 * dp + 1], pa, bb1);
      }
    }
    __syncthreads();  // every warp is done with this stage (and with conv_buf)
    if (tid == 0 && produce(stage)) ++produced;

    if (m.last) {
      // merge the 4 warps' partial softmax states of this item and store it
      float lsum[2] = {lrow[0], lrow[1]};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        lsum[r] += __shfl_xor_sync(0xffffffffu, lsum[r], 1);
        lsum[r] += __shfl_xor_sync(0xffffffffu, lsum[r], 2);
      }
      float* mw = merge + warp * g * MLD;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + 2 * (lane & 3);
        if (ra < g) {
          mw[ra * MLD + col] = acc[nt][0];
          mw[ra * MLD + col + 1] = acc[nt][1];
        }
        if (rb < g) {
          mw[rb * MLD + col] = acc[nt][2];
          mw[rb * MLD + col + 1] = acc[nt][3];
        }
      }
      if ((lane & 3) == 0) {
        if (ra < g) {
          mw[ra * MLD + D] = mrow[0];
          mw[ra * MLD + D + 1] = lsum[0];
        }
        if (rb < g) {
          mw[rb * MLD + D] = mrow[1];
          mw[rb * MLD + D + 1] = lsum[1];
        }
      }
      __syncthreads();
      const float vscale = FP8 ? c.v_scale[m.page] : 1.0f;
      for (int idx = tid; idx < g * (D + 1); idx += 128) {
        const int r = idx / (D + 1), d = idx % (D + 1);
        float M = -INFINITY;
        for (int wv = 0; wv < 4; ++wv) M = fmaxf(M, merge[(wv * g + r) * MLD + D]);
        const float Mu = M == -INFINITY ? 0.f : M;
        float sum = 0.f;
        for (int wv = 0; wv < 4; ++wv) {
          const float f = exp2f(merge[(wv * g + r) * MLD + D] - Mu);
          sum += f * merge[(wv * g + r) * MLD + (d < D ? d : D + 1)];
        }
        if (d < D) {
          c.part_acc[(static_cast<long>(m.item) * g + r) * D + d] = sum * vscale;
        } else {
          c.part_ml[(static_cast<long>(m.item) * g + r) * 2] = M;
          c.part_ml[(static_cast<long>(m.item) * g + r) * 2 + 1] = sum;
        }
      }
      cur_item = -1;
    }
  }
}

// LSE combine of the partials of each head: o = sum_i 2^(m_i - M) acc_i / sum_i 2^(m_i - M) l_i.
template <typename TO>
__global__ void k_decode_combine(CacheView c, int layer, TO* o) {
  const int hq = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int g = c.Hq / c.Hkv, h = hq / g, r = hq % g, D = c.D;
  const int bh = b * c.Hkv + h;
  const int i0 = c.item_off[bh], i1 = c.item_off[bh + 1];
  float M = -INFINITY;
  for (int i = i0; i < i1; ++i) M = fmaxf(M, c.part_ml[(static_cast<long>(i) * g + r) * 2]);
  const float Mu = M == -INFINITY ? 0.f : M;
  float L = 0.f, acc = 0.f;
  for (int i = i0; i < i1; ++i) {
    const float f = exp2f(c.part_ml[(static_cast<long>(i) * g + r) * 2] - Mu);
    L += f * c.part_ml[(static_cast<long>(i) * g + r) * 2 + 1];
    acc += f * c.part_acc[(static_cast<long>(i) * g + r) * D + d];
  }
  if (d < D) o[(static_cast<long>(b) * c.Hq + hq) * D + d] = from_f<TO>(L > 0.f ? acc / L : 0.f);
}

template <int D, bool FP8>
static cudaError_t launch_attn(const CacheView& c, int layer, const void* q, void* o, const CUtensorMap* kmap,
                               const CUtensorMap* vmap, int num_sms, cudaStream_t s) {
  using S = DecodeSmem<D, FP8>;
  const int g = c.Hq / c.Hkv;
  const size_t smem = 1024 + kStages * S::STAGE + S::CONV + 4 * g * (D + 2) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_decode_attn<D, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = 2 * num_sms;
  k_decode_attn<D, FP8><<<grid, 128, smem, s>>>(c, layer, static_cast<const __nv_bfloat16*>(q), *kmap, *vmap);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 cg(c.Hq, c.B);
  k_decode_combine<__nv_bfloat16><<<cg, D, 0, s>>>(c, layer, static_cast<__nv_bfloat16*>(o));
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
