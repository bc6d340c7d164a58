// Decode attention with one thread-block cluster per KV head, and the fused
// decode step built on it.
//
// A cluster of `cs` CTAs (cs a power of two <= 8, chosen so the grid holds
// about two CTAs per SM) covers one (b, h): CTA r attends a contiguous range of
// the head's retained slots, staged by TMA in sub-tiles of at most 64 slots
// that never cross a page, with the g query heads as the M dimension of
// mma.sync tiles.  Each CTA leaves its merged partial (acc, running max,
// running sum, log2 domain) in its own shared memory; after a cluster barrier
// rank 0 reads the cs partials through distributed shared memory and writes
// the head's output rows ([FastDMS], attention scoring: split-K grouped compact
// decode attention over variable-length per-head live spans -- here the split
// never leaves the chip).
//
// FUSED (bf16 pages): the whole decode step in one launch.  The attention runs
// over the slots as they were before this step's append, with the slot this
// token reuses masked out and the new token's key/value taken from the input
// as one more key of rank 0 -- the same visible set as after the append.  Rank
// 0 then appends the token at the slot fixed by the plan of the previous step
// ([DMS-Qwen3], inference mode: a token overwrites the slot of the token
// leaving the window when that one was marked, else takes the next slot; a new
// page when that slot starts one), updates the head's count and writes the
// plan of the next append.  New pages are numbered from the page counter as
// read at the start plus the head's rank among the heads needing one, i.e. in
// (b, h) row-major order; the grid's last CTA advances the counter and the
// positions.
#include "decode_common.cuh"

namespace dms {

#ifdef DMS_TRACE
__device__ unsigned long long g_dms_trace[2 * kTraceCtas * kTraceSlots];
#endif

constexpr int kMaxCluster = 16;  // shared-memory staging bound
constexpr int kPickCluster = 8;  // largest cluster launched: every cluster of the grid co-resident

template <int D, bool FP8>
struct ClusterSmem {
  using S = DecodeSmem<D, FP8>;
  static constexpr int MLD = D + 2;
  static size_t bytes(int g) {
    return 1024 + kStages * S::STAGE + S::CONV + (5 * g + g) * MLD * sizeof(float) +
           (3 * kMaxCluster * 16 + 16) * sizeof(float);
  }
};

struct SubMeta {
  int slot;  // first slot of the sub-tile
  int rows;  // slots in the sub-tile (<= 64, inside one page)
  int page;  // page id
};

template <int D, bool FP8, bool FUSED>
__global__ void __launch_bounds__(kThreads) k_decode_cluster(CacheView c, int layer, const __nv_bfloat16* q,
                                                            __nv_bfloat16* o, int cs, const __nv_bfloat16* k_new,
                                                            const __nv_bfloat16* v_new, float* alpha, DecideArgs da,
                                                            int fuse_decide,
                                                            const __grid_constant__ CUtensorMap kmap,
                                                            const __grid_constant__ CUtensorMap vmap) {
  using S = DecodeSmem<D, FP8>;
  constexpr int KS = D / 16, NT = D / 8, MLD = D + 2;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sbase =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* stage_buf = sbase;
  unsigned char* conv_buf = sbase + kStages * S::STAGE;
  const int g = c.Hq / c.Hkv;
  float* merge = reinterpret_cast<float*>(conv_buf + S::CONV);  // [5 sources][g][MLD]
  float* cpart = merge + 5 * g * MLD;                           // [g][MLD] this CTA's partial
  float* sm_m = cpart + g * MLD;                                // [cs][g] maxima of the cluster's partials
  float* sm_l = sm_m + kMaxCluster * 16;                        // [cs][g] sums, then weights
  float* sm_w = sm_l + kMaxCluster * 16;                        // [cs][g] weights
  float* sm_L = sm_w + kMaxCluster * 16;                        // [g]
  __shared__ uint64_t full_bar[kStages];
  __shared__ SubMeta meta[kStages];
  __shared__ int s_abort, s_have, s_last, s_red[32], s_ring_next;
  __shared__ float s_fred[8], s_alpha, s_xscore[16];
  __shared__ __align__(16) __nv_bfloat16 s_knew[D], s_vnew[D];
  constexpr int kPtCache = 256;  // page-table entries of the head kept in shared memory
  __shared__ int s_pt[kPtCache];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / cs;
  const int rank = static_cast<int>(cluster_rank());
  const int owner = cs - 1;  // the rank that appends: its slice of the slots is the shortest
  const int b = bh / c.Hkv, h = bh % c.Hkv;
  const long li = static_cast<long>(layer) * c.B * c.Hkv + bh;
  DMS_TRACE_MARK(0, 0);
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&full_bar[i], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  // state of this head (stable during the launch: only rank 0 of this head's
  // cluster writes it, after the cluster barrier; the position and the page
  // counter only change in the grid's last CTA)
  // the head's page-table row is fetched together with the count (no dependent round trip)
  for (int i = tid; i < min(c.maxp, kPtCache); i += kThreads) s_pt[i] = c.page_table[li * c.maxp + i];
  const int cnt = c.count[li];
  const int t = FUSED ? c.pos[layer * c.B + b] : 0;
  const int4 pl = FUSED ? *plan_at(c, li, t) : make_int4(0, 0, 0, 0);
  const int masked_slot = (FUSED && (pl.y & 1)) ? pl.x : -1;
  const int next_page0 = FUSED ? c.ctrl[CTRL_NEXT_PAGE] : 0;
  const int per = ((cnt + cs - 1) / cs + 15) / 16 * 16;
  const int s_begin = min(cnt, rank * per), s_end = min(cnt, s_begin + per);
  __syncthreads();

  int p_s = s_begin;
  auto produce = [&](int stage) -> bool {
    if (p_s >= s_end) return false;
    const int pi = p_s / c.P;
    const int page = pi < kPtCache ? s_pt[pi] : c.page_table[li * c.maxp + pi];
    const int rows = min(min(kSub, s_end - p_s), c.P - p_s % c.P);
    meta[stage].slot = p_s;
    meta[stage].rows = rows;
    meta[stage].page = page;
    issue_subtile<D, FP8>(stage_buf + stage * S::STAGE, &kmap, &vmap, page * c.P + p_s % c.P, rows, &full_bar[stage]);
    p_s += rows;
    return true;
  };
  int produced = 0;
  if (tid == 0)
    for (int st = 0; st < kStages; ++st)
      if (produce(st)) ++produced;

  uint32_t qa[KS][4];
  const __nv_bfloat16* qb = q + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D;
  load_q_frags<D>(qb, g, qa);
  if (FUSED && rank == owner) {
    // everything the append needs, fetched while the first tiles are in flight:
    // the new key/value row, the new token's scores, the ring entry of t + 1
    if (tid < D / 8) {
      reinterpret_cast<uint4*>(s_knew)[tid] = reinterpret_cast<const uint4*>(k_new + static_cast<long>(bh) * D)[tid];
      reinterpret_cast<uint4*>(s_vnew)[tid] = reinterpret_cast<const uint4*>(v_new + static_cast<long>(bh) * D)[tid];
    }
    if (tid == 32) s_ring_next = (t + 1 >= c.w) ? c.ring[li * c.w + (t + 1) % c.w] : 0;
    __syncthreads();
    for (int r = warp; r < g; r += 4) {
      float sdot = 0.f;
      for (int d = lane; d < D; d += 32)
        sdot = fmaf(__bfloat162float(qb[static_cast<long>(r) * D + d]), __bfloat162float(s_knew[d]), sdot);
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o2);
      if (lane == 0) s_xscore[r] = sdot;
    }
  }
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  if (FUSED && rank == owner && fuse_decide) {
    // decision logit of the new token (layer granularity: head 0's)
    const int src = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
    const float a = decide_cta<4>(c, da, b, src, s_fred);
    if (tid == 0) {
      s_alpha = a;
      alpha[b * c.Hkv + h] = a;
    }
  }

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
    const SubMeta m = meta[stage];
    if (n == 0) DMS_TRACE_MARK(0, 2);
    const unsigned char* kt = stage_buf + stage * S::STAGE;
    if (FP8) {
      widen_fp8_subtile<D>(kt, conv_buf);
      __syncthreads();
      kt = conv_buf;
    }
    const unsigned char* vt = kt + (FP8 ? S::TILE_BF16 : S::TILE_RAW);
    if (warp * 16 < m.rows) {
      const float kscale = FP8 ? c.k_scale[m.page] : 1.0f;
      const float vscale = FP8 ? c.v_scale[m.page] : 1.0f;
      warp_tile<D>(kt, vt, m.rows, masked_slot - m.slot, kscale * sl2, vscale, qa, acc, mrow, lrow);
    }
    __syncthreads();
    if (tid == 0 && produce(stage)) ++produced;
  }

  DMS_TRACE_MARK(0, 3);
  // merge the warps (and, for rank 0 of a fused step, the new token) into this
  // CTA's partial
  warp_state_to_smem<D>(merge, warp, g, acc, mrow, lrow);
  int nsrc = 4;
  if (FUSED && rank == owner) {
    // the new token as a fifth source: score q_r . k_new, weight 1, value v_new
    for (int r = tid; r < g; r += kThreads) {
      merge[(4 * g + r) * MLD + D] = s_xscore[r] * sl2;
      merge[(4 * g + r) * MLD + D + 1] = 1.0f;
    }
    for (int idx = tid; idx < g * D; idx += kThreads) merge[(4 * g + idx / D) * MLD + idx % D] = __bfloat162float(s_vnew[idx % D]);
    nsrc = 5;
  }
  __syncthreads();
  merge_sources<D>(merge, nsrc, g, 1.0f, [&](int r, int d, float v) { cpart[r * MLD + d] = v; });
  cluster_sync();  // every partial of the cluster is in place
  DMS_TRACE_MARK(0, 4);

  // Combine the cs partials through distributed shared memory: CTA `rank`
  // merges output elements [rank * per_cta, (rank + 1) * per_cta) of the head's
  // g x D block, with every remote load of a thread issued before use.
  {
    const int total = g * D;
    const int per_cta = (total + cs - 1) / cs;
    const int e0 = rank * per_cta, e1 = min(total, e0 + per_cta);
    const int r0 = e0 / D, r1 = e1 > e0 ? (e1 - 1) / D : r0 - 1;  // rows touched
    const int nrows = r1 - r0 + 1;
    for (int idx = tid; idx < cs * nrows; idx += kThreads) {
      const int k = idx / nrows, r = r0 + idx % nrows;
      sm_m[idx] = ld_dsmem(dsmem_addr(&cpart[r * MLD + D], k));
      sm_l[idx] = ld_dsmem(dsmem_addr(&cpart[r * MLD + D + 1], k));
    }
    __syncthreads();
    if (tid < nrows) {
      float M = -INFINITY;
      for (int k = 0; k < cs; ++k) M = fmaxf(M, sm_m[k * nrows + tid]);
      const float Mu = M == -INFINITY ? 0.f : M;
      float L = 0.f;
      for (int k = 0; k < cs; ++k) {
        const float wgt = exp2f(sm_m[k * nrows + tid] - Mu);
        sm_w[k * nrows + tid] = wgt;
        L += wgt * sm_l[k * nrows + tid];
      }
      sm_L[tid] = L;
    }
    __syncthreads();
    __nv_bfloat16* ob = o + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D;
    constexpr int EPT = 4;  // output elements per thread per pass
    for (int base = e0; base < e1; base += kThreads * EPT) {
      float v[EPT][kPickCluster];
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        const int e = base + j * kThreads + tid;
#pragma unroll
        for (int k = 0; k < kPickCluster; ++k)
          v[j][k] = (e < e1 && k < cs) ? ld_dsmem(dsmem_addr(&cpart[(e / D) * MLD + e % D], k)) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        const int e = base + j * kThreads + tid;
        if (e >= e1) continue;
        const int rl = e / D - r0;
        float a = 0.f;
#pragma unroll
        for (int k = 0; k < kPickCluster; ++k)
          if (k < cs) a = fmaf(sm_w[k * nrows + rl], v[j][k], a);
        const float L = sm_L[rl];
        ob[e] = __float2bfloat16_rn(L > 0.f ? a / L : 0.f);
      }
    }
  }

  if (rank == owner) {
    if (FUSED) {
      // append of this head's token at the planned slot (every CTA of the
      // cluster has finished reading the pages: cluster barrier above)
      const int flags = pl.y, slot = pl.x;
      int id = -1;
      bool ok = !(flags & 4);
      if (ok && (flags & 2)) {
        int n_before = 0;
        for (int i = tid; i < bh; i += kThreads)
          n_before += (plan_at(c, static_cast<long>(layer) * c.B * c.Hkv + i, t)->y & 2) ? 1 : 0;
        int before;
        block_exclusive_scan(n_before, s_red, &before);
        id = next_page0 + before;
        if (id >= c.pool_pages || c.npages[li] >= c.maxp) ok = false;
      } else if (ok) {
        id = c.page_table[li * c.maxp + slot / c.P];
      }
      int cnt_new = cnt, np_new = c.npages[li];
      if (ok) {
        const long row = static_cast<long>(id) * c.P + slot % c.P;
        if (tid < D / 8) {
          reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.k_pool) + row * D)[tid] =
              reinterpret_cast<const uint4*>(s_knew)[tid];
          reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.v_pool) + row * D)[tid] =
              reinterpret_cast<const uint4*>(s_vnew)[tid];
        }
        if (!(flags & 1)) cnt_new = cnt + 1;
        if (flags & 2) np_new += 1;
        if (tid == 0) {
          if (flags & 2) {
            c.page_table[li * c.maxp + np_new - 1] = id;
            c.npages[li] = np_new;
            atomicAdd(&c.ctrl[CTRL_STEP_PAGES], 1);
          }
          const int hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
          const float a = fuse_decide ? s_alpha : __ldcg(&alpha[b * c.Hkv + hs]);
          const bool evict = !c.disable && a > 0.0f;
          c.slot_pos[li * c.cap + slot] = t;
          c.ring[li * c.w + t % c.w] = slot | (evict ? static_cast<int>(RING_EVICT) : 0);
          if (!(flags & 1)) c.count[li] = cnt_new;
        }
      } else if (tid == 0) {
        set_status(c.ctrl, (flags & 4) ? DMS_ST_CAPACITY : DMS_ST_POOL_EXHAUSTED);
      }
      if (tid == 0) {
        // plan of the next append (token t + 1), from the values just written
        *plan_at(c, li, t + 1) = make_plan(s_ring_next, t + 1, cnt_new, np_new, c);
      }
    }
  }
  DMS_TRACE_MARK(0, 5);
  cluster_sync();  // rank 0 is done reading the cluster's shared memory

  if (FUSED) {
    // the grid's last CTA advances the page counter and the positions
    if (tid == 0) {
      __threadfence();
      s_last = (atomicAdd(&c.ctrl[CTRL_GRID_DONE], 1) == static_cast<int>(gridDim.x) - 1) ? 1 : 0;
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      if (tid == 0) {
        const int granted = __ldcg(&c.ctrl[CTRL_STEP_PAGES]);
        c.ctrl[CTRL_NEXT_PAGE] = min(__ldcg(&c.ctrl[CTRL_NEXT_PAGE]) + granted, c.pool_pages);
        c.ctrl[CTRL_STEP_PAGES] = 0;
        c.ctrl[CTRL_GRID_DONE] = 0;
      }
      for (int bb = tid; bb < c.B; bb += kThreads) c.pos[layer * c.B + bb] += 1;
    }
  }
  DMS_TRACE_MARK(0, 6);
}

// Cluster size: the largest power of two <= 8 with cs * B * Hkv <= 2 * SMs
// (about two CTAs per SM) that the device can co-schedule.
template <int D, bool FP8, bool FUSED>
static int pick_cluster(int heads, int num_sms, size_t smem) {
  static int max_cs = 0;
  if (max_cs == 0) {
    max_cs = 1;
    for (int cs = kPickCluster; cs > 1; cs >>= 1) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(cs, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k_decode_cluster<D, FP8, FUSED>, &cfg) == cudaSuccess && n > 0) {
        max_cs = cs;
        break;
      }
      cudaGetLastError();
    }
  }
  int cs = 1;
  while (cs * 2 <= max_cs && static_cast<long>(cs) * 2 * heads <= 2L * num_sms) cs *= 2;
  return cs;
}

template <int D, bool FP8, bool FUSED>
static cudaError_t launch_cluster_t(const CacheView& c, int layer, const void* q, void* o, const void* k,
                                   const void* v, float* alpha, const DecideArgs* da, const CUtensorMap* kmap,
                                   const CUtensorMap* vmap, int num_sms, cudaStream_t s) {
  const int g = c.Hq / c.Hkv;
  const size_t smem = ClusterSmem<D, FP8>::bytes(g);
  auto kern = k_decode_cluster<D, FP8, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  const int heads = c.B * c.Hkv;
  const int cs = pick_cluster<D, FP8, FUSED>(heads, num_sms, smem);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(cs * heads, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  DecideArgs none{};
  return cudaLaunchKernelEx(&cfg, kern, c, layer, static_cast<const __nv_bfloat16*>(q),
                            static_cast<__nv_bfloat16*>(o), cs, static_cast<const __nv_bfloat16*>(k),
                            static_cast<const __nv_bfloat16*>(v), alpha, da ? *da : none, da ? 1 : 0, *kmap, *vmap);
}

cudaError_t launch_decode_cluster(const CacheView& c, int layer, const void* q, void* o, bool fused, const void* k,
                                  const void* v, float* alpha, const DecideArgs* fused_decide, const CUtensorMap* kmap,
                                  const CUtensorMap* vmap, int num_sms, cudaStream_t s) {
  if (!kmap || !vmap || c.kv_dtype == DMS_F32) return cudaErrorInvalidValue;
  if (fused) {
    if (c.kv_dtype != DMS_BF16) return cudaErrorInvalidValue;
    return c.D == 64 ? launch_cluster_t<64, false, true>(c, layer, q, o, k, v, alpha, fused_decide, kmap, vmap, num_sms, s)
                     : launch_cluster_t<128, false, true>(c, layer, q, o, k, v, alpha, fused_decide, kmap, vmap, num_sms, s);
  }
  if (c.kv_dtype == DMS_FP8_E4M3)
    return c.D == 64 ? launch_cluster_t<64, true, false>(c, layer, q, o, k, v, alpha, nullptr, kmap, vmap, num_sms, s)
                     : launch_cluster_t<128, true, false>(c, layer, q, o, k, v, alpha, nullptr, kmap, vmap, num_sms, s);
  return c.D == 64 ? launch_cluster_t<64, false, false>(c, layer, q, o, k, v, alpha, nullptr, kmap, vmap, num_sms, s)
                   : launch_cluster_t<128, false, false>(c, layer, q, o, k, v, alpha, nullptr, kmap, vmap, num_sms, s);
}

}  // namespace dms

#ifdef DMS_TRACE
// Copy the cluster kernel's phase timeline to the host (tracing builds only).
extern "C" __attribute__((visibility("default"))) int dms_debug_trace_read_cluster(void* host, size_t bytes) {
  const size_t n = sizeof(dms::g_dms_trace) < bytes ? sizeof(dms::g_dms_trace) : bytes;
  return cudaMemcpyFromSymbol(host, dms::g_dms_trace, n) == cudaSuccess ? 0 : -3;
}
#endif
