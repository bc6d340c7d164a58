// Decode attention as one persistent split-K pass over every head's retained
// slots, balanced across all SMs, and the fused decode step built on it.
//
// Work: the retained slots of all (b, h) of a layer, cut into units of 16 * 2^k
// slots (every head gets at least one unit; k is the smallest leaving each CTA
// at most 62 units), laid end to end; CTA i of the G CTAs (one per SM) takes
// units [i*U/G, (i+1)*U/G).  Its range covers the tail of one head, whole
// heads, and the start of another ("segments").  A producer warp streams the
// range through a ring of shared-memory stages with TMA, one 32-slot sub-tile
// per stage (never crossing a page; one 32-row box per 128-byte column half of
// K and of V, plus the head's query rows).  Sub-tile n is consumed by consumer
// warp n mod 4 from one of that warp's own stages (stage w + 4 * (n/4 mod m),
// m stages per warp, so every use of a stage is ordered by the one warp that
// waits on it and no mbarrier is ever waited on two phases ahead), and the
// warp runs the whole online-softmax update of its keys on mma.sync tiles
// (keys as the M dimension and the g <= 8 query heads as N, else the
// reverse); the four warps' states are merged at the end of each segment
// ([FastDMS], attention
// scoring: split-K grouped decode attention over variable-length per-head
// spans; the balanced flat split keeps every SM streaming whatever the batch
// and the retained lengths).
//
// A head held by one CTA is finished there.  A head shared by n CTAs leaves n
// partials (acc, running max, running sum; log2 domain) in global scratch;
// the CTA whose arrival completes the head's counter merges them (LSE
// combine) and writes the output rows.  The consumers only merge their four
// warp states at a segment's end and hand the result to an aux warp through a
// two-deep ring; the aux warp writes partials, counts arrivals and finishes
// heads while the consumers stream on.
//
// FUSED (bf16 pages): the whole decode step in this launch, as in the cluster
// kernel.  The attention covers the slots as they were before this step's
// append, with the slot this token reuses excluded, plus the new token's
// key/value taken from the input as one more key, merged in by the finishing
// CTA -- the same visible set as after the append ([DMS-Qwen3], inference
// mode).  Every count the partition uses is the snapshot in the append plan,
// which no CTA of this launch rewrites.  The CTA holding a head's first unit
// computes the head's decision logit while its first tiles land; the
// finishing CTA appends the token at the slot planned by the previous step,
// updates the head's count, grants a page when the slot starts one (ids: the
// page counter at launch plus the head's rank among the heads needing one,
// (b, h) row-major) and writes the plan of the next append.  The grid's last
// CTA advances the page counter and the positions.
#include <algorithm>

#include "decode_common.cuh"

namespace dms {


constexpr int kFlatConsumers = 4;                        // warps computing
constexpr int kFlatProducer = kFlatConsumers;            // warp issuing the TMA loads
constexpr int kFlatAux = kFlatConsumers + 1;             // warp preparing the append
constexpr int kFlatThreads = (kFlatConsumers + 2) * 32;
constexpr int kFlatPrefetch = 8;                         // segments whose new K/V rows are staged
constexpr int kFlatUnit = 16;                            // slots per work unit (smallest)
constexpr int kFlatSegMax = 64;                          // head segments per CTA
constexpr int kFlatPtMax = 512;                          // page ids staged per CTA
constexpr int kFlatSubMax = 256;                         // sub-tile descriptors staged per CTA
constexpr int kFlatMaxStages = 16;
constexpr int kFlatRows = 32;                            // slots per sub-tile = rows per TMA box

struct FlatSeg {
  int bh;           // head, b * Hkv + h
  int s0, s1;       // this CTA's slots of the head
  int n0, n1;       // this CTA's sub-tiles [n0, n1) holding them
  int nparts;       // CTAs sharing the head
  int first_cta;    // the first of them
  int first_pslot;  // partial slot of the first of them
  int pslot;        // this CTA's partial slot
  int unit0;        // first unit of the head
  int pt0;          // first page id of [s0, s1) in s_pt, -1: read from the page table
  int decide;       // 1: this CTA computes the head's decision logit
  int t;            // position of the token appended by this step
  int plx, ply;     // plan of the append: slot, flags (1 reuse, 2 new page, 4 over capacity)
  int cnt, npages;  // the head's retained slots and pages before the append
  int grant;        // rank of the head among those taking a new page this step
  int sp_idx;       // index in s_pt of the page of a reused slot, -1: none staged
  int ring_idx;     // index in s_ring of the ring entry of position t + 1 - w, -1: none
  int qoff;         // element offset of the head's query rows in q
};

// Stage and use count of sub-tile n: consumer warp n % 4 owns stages
// w, w + 4, ..., w + 4 (m - 1) and takes them in turn.
__device__ __forceinline__ void flat_stage(int n, int m, int* st, int* use) {
  const int j = n / kFlatConsumers;
  *st = n % kFlatConsumers + kFlatConsumers * (j % m);
  *use = j / m;
}

struct FlatMeta {
  int slot;  // first slot of the sub-tile
  int rows;  // slots in the sub-tile (0: an empty segment)
  float ks;  // FP8 page scales
  float vs;
};

// Contiguous global -> shared copy completing on `bar` (no multicast).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Barrier of the four consumer warps only (the producer warp never joins).
__device__ __forceinline__ void consumers_sync() { asm volatile("barrier.sync 1, 128;\n" ::: "memory"); }

// Adapter decision logit of the new token of sequence b for head `src`, by
// one warp (eight 16-byte vectors of each operand in flight per lane).
__device__ __forceinline__ float decide_warp(const CacheView& c, const DecideArgs& a, int b, int src) {
  const int lane = threadIdx.x & 31;
  const int hid = c.hidden, nvec = hid / 8;
  const uint4* xr =
      reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.hidden) + static_cast<long>(b) * hid);
  const uint4* wr =
      reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.W) + static_cast<long>(src) * hid);
  constexpr int VPT = 8;
  float ss = 0.f, dot = 0.f;
  for (int v0 = 0; v0 < nvec; v0 += 32 * VPT) {
    uint4 xu[VPT], wu[VPT], gu[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int vi = v0 + u * 32 + lane;
      const bool ok = vi < nvec;
      xu[u] = ok ? xr[vi] : make_uint4(0, 0, 0, 0);
      wu[u] = ok ? wr[vi] : make_uint4(0, 0, 0, 0);
      gu[u] = ok ? gamma16<__nv_bfloat16>(a.gamma, vi) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
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
  const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(a.bias);
  return adapter_logit(c, dot, ss, hid, bias ? __bfloat162float(bias[src]) : 0.f, a.offset[b * a.offset_bstride + src]);
}

template <int D, bool FP8>
struct FlatSmem {
  static constexpr int HALVES = D / 64;
  static constexpr int TILE = FP8 ? kFlatRows * D : HALVES * kFlatRows * 128;  // K (or V) of one sub-tile
  static constexpr int CROWS = kFlatRows;                                      // FP8 rows widened at a time
  static constexpr int CONV_WARP = FP8 ? 2 * CROWS * D * 2 : 0;                // K + V widened, per warp
  static constexpr int MLD = D + 2;
  __host__ __device__ static size_t stage_stride(int g) {
    return (static_cast<size_t>(2 * TILE) + g * D * 2 + 1023) / 1024 * 1024;
  }
  // everything but the stage ring
  __host__ __device__ static size_t fixed(int g) {
    return 1024 + static_cast<size_t>(kFlatConsumers) * CONV_WARP + (4 * g + 2 * g) * MLD * sizeof(float);
  }
};

template <int D, bool FP8, bool FUSED, bool TQ>
__global__ void __launch_bounds__(kFlatThreads, 1)
    k_decode_flat(CacheView c, int layer, int early, const __nv_bfloat16* q, __nv_bfloat16* o, int nst,
                  const __nv_bfloat16* k_new, const __nv_bfloat16* v_new, float* alpha, DecideArgs da, int fuse_decide,
                  const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
  using F = FlatSmem<D, FP8>;
  constexpr int KS = D / 16, NT = D / 8, MLD = D + 2;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sbase =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int g = c.Hq / c.Hkv;
  const size_t stride = F::stage_stride(g);
  unsigned char* conv_buf = sbase + nst * stride;                                     // [warp][K, V] (FP8)
  float* merge = reinterpret_cast<float*>(conv_buf + kFlatConsumers * F::CONV_WARP);  // [4 warps][g][MLD]
  float* cpart = merge + 4 * g * MLD;  // [2][g][MLD] merged segments handed to the aux warp
  __shared__ uint64_t full_bar[kFlatMaxStages], empty_bar[kFlatMaxStages];
  __shared__ FlatMeta meta[kFlatMaxStages];
  __shared__ FlatSeg segs[kFlatSegMax];
  __shared__ int s_pt[kFlatPtMax];
  __shared__ long s_ptsrc[kFlatPtMax];
  __shared__ int4 s_sub[kFlatSubMax];                               // sub-tile descriptors
  __shared__ int s_n0[kFlatSegMax];                                 // first sub-tile of each segment
  __shared__ float s_ks[FP8 ? kFlatSubMax : 1], s_vs[FP8 ? kFlatSubMax : 1];  // FP8 scales per sub-tile
  __shared__ int s_ring[kFlatSegMax];
  __shared__ long s_ringsrc[kFlatSegMax];
  __shared__ float s_x[FUSED ? kFlatSegMax : 1][16];  // new token's scores per segment
  __shared__ float s_alpha[FUSED ? kFlatSegMax : 1];   // new token's decision logit per segment
  __shared__ __align__(16) __nv_bfloat16 s_kvnew[FUSED ? kFlatPrefetch : 1][2][D];  // new K, V rows
  __shared__ __align__(8) uint64_t hq_full[2], hq_empty[2];  // merged-segment hand-over ring
  __shared__ __align__(8) uint64_t aux_done;                 // every hand-over processed
  __shared__ int s_fin[kFlatSegMax], s_nfin;                 // heads the consumers finish
  __shared__ int s_part[kFlatThreads / 32][8];  // per-warp candidate unit sums
  __shared__ int s_ctot[kFlatThreads / 32][2];  // per-warp chunk totals (units, new pages)
  __shared__ int s_stot[2][3];                  // per-warp segment totals (sub-tiles, page ids, ring entries)
  __shared__ int s_nseg, s_nsub, s_npt, s_nring, s_last, s_next_page0, s_grants;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int BH = c.B * c.Hkv;
  const long lbase = static_cast<long>(layer) * BH;
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  // Programmatic dependent launch.  With `early` (the previous launch of this
  // library on the stream was for another layer or cache) the partition below
  // reads only this layer's state before waiting for the previous kernel:
  // only that kernel may still run (each kernel lets its dependents start
  // only once its own wait has returned), and it does not write this state.
  // The page counter, the arrival counters, the partial scratch and the
  // inputs are touched only after the wait.
  if (!early) {
    griddep_wait();
    griddep_launch_dependents();
  }

  // ---- setup: every CTA derives the same partition ------------------------
  // (scratch arrays live in the stage ring, unused until the producer starts)
  int* s_cnt = reinterpret_cast<int*>(sbase);
  int* s_off = s_cnt + BH;     // [BH + 1] unit offsets
  int* s_gr = s_off + BH + 1;  // [BH] new-page ranks
  int* s_plx = s_gr + BH;      // [BH] plan slot
  int* s_ply = s_plx + BH;     // [BH] plan flags
  int* s_npg = s_ply + BH;     // [BH] pages before the append
  int* s_tpos = s_npg + BH;    // [BH] position of the appended token
  if (warp == kFlatProducer && lane == 0) {
    // the TMA descriptors, fetched while the partition is worked out
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < nst; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&hq_full[i], 1);
      mbar_init(&hq_empty[i], 1);
    }
    mbar_init(&aux_done, 1);
    s_nfin = 0;
    s_grants = 0;
    fence_mbar_init();
  }
  // Heads are split into one contiguous chunk per warp.  Each warp loads its
  // chunk's plans (both parities and the position in one round trip); warp
  // shuffles then do the reductions and scans, with one exchange of chunk
  // totals between the warps.
  constexpr int NW = kFlatThreads / 32;
  const int hchunk = (BH + NW - 1) / NW;
  const int hb = min(BH, warp * hchunk), he = min(BH, hb + hchunk);
  {
    int part[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    constexpr int LB = 4;  // heads per lane whose loads are in flight together
    for (int i0 = hb; i0 < he; i0 += 32 * LB) {
      int4 pa[LB], pb[LB];
      int tt[LB], cc[LB];
#pragma unroll
      for (int u = 0; u < LB; ++u) {
        const int i = i0 + u * 32 + lane;
        if (i < he) {
          if (FUSED) {
            pa[u] = c.plan[lbase + i];
            pb[u] = c.plan[static_cast<long>(c.L) * BH + lbase + i];
            tt[u] = c.pos[layer * c.B + i / c.Hkv];
          } else {
            cc[u] = c.count[lbase + i];  // nothing in this launch changes it
          }
        }
      }
#pragma unroll
      for (int u = 0; u < LB; ++u) {
        const int i = i0 + u * 32 + lane;
        if (i >= he) continue;
        int cnt;
        if (FUSED) {
          // the plan of position t holds the count before this step's append
          const int4 pl = (tt[u] & 1) ? pb[u] : pa[u];
          cnt = pl.z;
          s_plx[i] = pl.x;
          s_ply[i] = pl.y;
          s_npg[i] = pl.w;
          s_tpos[i] = tt[u];
        } else {
          cnt = cc[u];
        }
        s_cnt[i] = cnt;
#pragma unroll
        for (int k = 0; k < 8; ++k) part[k] += max(1, (cnt + (kFlatUnit << k) - 1) / (kFlatUnit << k));
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) part[k] += __shfl_xor_sync(0xffffffffu, part[k], o2);
    if (lane == 0)
#pragma unroll
      for (int k = 0; k < 8; ++k) s_part[warp][k] = part[k];
  }
  __syncthreads();
  // unit size (every thread alike): the smallest 16 * 2^k slots leaving at
  // most kFlatSegMax - 2 units per CTA, so a CTA's range meets at most that
  // many heads
  int unit = kFlatUnit;
  for (int k = 0;; ++k) {
    long tot = 0;
#pragma unroll
    for (int wv = 0; wv < NW; ++wv) tot += s_part[wv][k];
    unit = kFlatUnit << k;
    if (k == 7 || (tot + G - 1) / G <= kFlatSegMax - 2) break;
  }
  // unit offsets and new-page ranks: scans within each warp's chunk
  {
    int carry = 0, gcarry = 0;
    for (int i0 = hb; i0 < he; i0 += 32) {
      const int i = i0 + lane;
      const int n = i < he ? max(1, (s_cnt[i] + unit - 1) / unit) : 0;
      const int np = (FUSED && i < he && (s_ply[i] & 2)) ? 1 : 0;
      int x = n, y = np;
#pragma unroll
      for (int o2 = 1; o2 < 32; o2 <<= 1) {
        const int xa = __shfl_up_sync(0xffffffffu, x, o2), ya = __shfl_up_sync(0xffffffffu, y, o2);
        if (lane >= o2) {
          x += xa;
          y += ya;
        }
      }
      if (i < he) {
        s_off[i] = carry + x - n;
        if (FUSED) s_gr[i] = gcarry + y - np;
      }
      carry += __shfl_sync(0xffffffffu, x, 31);
      gcarry += __shfl_sync(0xffffffffu, y, 31);
    }
    if (lane == 0) {
      s_ctot[warp][0] = carry;
      s_ctot[warp][1] = gcarry;
    }
  }
  __syncthreads();
  {
    int base = 0, gbase = 0, total = 0;
#pragma unroll
    for (int wv = 0; wv < NW; ++wv) {
      if (wv < warp) {
        base += s_ctot[wv][0];
        gbase += s_ctot[wv][1];
      }
      total += s_ctot[wv][0];
    }
    for (int i = hb + lane; i < he; i += 32) {
      s_off[i] += base;
      if (FUSED) s_gr[i] += gbase;
    }
    if (tid == 0) s_off[BH] = total;
  }
  __syncthreads();
  const long U = s_off[BH];
  const long u0 = static_cast<long>(cta) * U / G, u1 = static_cast<long>(cta + 1) * U / G;
  auto cta_of = [&](long u) {
    const unsigned long long a = static_cast<unsigned long long>(u + 1) * G - 1;
    return static_cast<int>((a >> 32) == 0 && (U >> 32) == 0 ? static_cast<unsigned>(a) / static_cast<unsigned>(U)
                                                              : a / static_cast<unsigned long long>(U));
  };
  // heads [h_lo, h_hi] meet this CTA's units (binary searches in every thread)
  int h_lo = 0, h_hi = -1;
  if (u0 < u1) {
    int lo = 0, hi = BH - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= u0) lo = mid; else hi = mid - 1;
    }
    h_lo = lo;
    hi = BH - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] < u1) lo = mid; else hi = mid - 1;
    }
    h_hi = lo;
  }
  int nseg = h_hi - h_lo + 1;
  if (nseg > kFlatSegMax) {
    if (tid == 0) set_status(c.ctrl, DMS_ST_SPLIT_LIMIT);
    nseg = kFlatSegMax;
  }
  const int chunk = c.P % kFlatRows == 0 ? kFlatRows : 16;
  // segments: warps 0 and 1, one lane per segment (kFlatSegMax = 64); their
  // sub-tile, page-id and ring-entry counts are scanned with shuffles
  FlatSeg sg{};
  int my_sub = 0, my_pt = 0, my_ring = 0, p0 = 0, p1 = -1;
  int xs = 0, xp = 0, xr = 0;  // inclusive scans within the warp
  long li = 0;
  const int ks = warp * 32 + lane;
  if (warp < 2) {
    if (ks < nseg) {
      const int h = h_lo + ks;
      const int cnt = s_cnt[h];
      li = lbase + h;
      sg.bh = h;
      sg.cnt = cnt;
      sg.s0 = static_cast<int>(max(0L, u0 - s_off[h]) * unit);
      sg.s1 = static_cast<int>(min(static_cast<long>(cnt), (u1 - s_off[h]) * unit));
      if (sg.s0 > sg.s1) sg.s0 = sg.s1;  // an empty head's only unit
      sg.unit0 = s_off[h];
      if (s_off[h] >= u0 && s_off[h + 1] <= u1) {
        sg.nparts = 1;  // the whole head is here
        sg.first_cta = cta;
        sg.first_pslot = sg.pslot = 2 * cta;
      } else {
        const int fc = cta_of(s_off[h]), lc = cta_of(s_off[h + 1] - 1);
        sg.first_cta = fc;
        // with fewer units than CTAs most CTAs are empty: the head's parts are
        // then the CTAs of its units, one unit each
        sg.nparts = min(lc - fc + 1, s_off[h + 1] - s_off[h]);
        const long fu0 = static_cast<long>(fc) * U / G;
        sg.first_pslot = 2 * fc + (s_off[h] != fu0 ? 1 : 0);
        sg.pslot = cta == fc ? sg.first_pslot : 2 * cta;
      }
      sg.decide = (FUSED && fuse_decide && s_off[h] >= u0) ? 1 : 0;
      const int b = h / c.Hkv;
      sg.t = FUSED ? s_tpos[h] : 0;
      sg.plx = FUSED ? s_plx[h] : 0;
      sg.ply = FUSED ? s_ply[h] : 0;
      sg.npages = FUSED ? s_npg[h] : 0;
      sg.grant = FUSED ? s_gr[h] : 0;
      sg.qoff = (b * c.Hq + (h % c.Hkv) * g) * D;
      if (sg.s1 > sg.s0) {
        p0 = sg.s0 / c.P;
        p1 = (sg.s1 - 1) / c.P;
        my_sub = (sg.s1 - 1) / chunk - sg.s0 / chunk + 1;
        my_pt = p1 - p0 + 1;
      } else {
        my_sub = 1;  // one empty sub-tile carries the segment's end
      }
      if (FUSED && (sg.ply & 1)) ++my_pt;  // page of the reused slot
      my_ring = (FUSED && sg.t + 1 >= c.w) ? 1 : 0;
    }
    xs = my_sub;
    xp = my_pt;
    xr = my_ring;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
      const int a1 = __shfl_up_sync(0xffffffffu, xs, o2), a2 = __shfl_up_sync(0xffffffffu, xp, o2),
                a3 = __shfl_up_sync(0xffffffffu, xr, o2);
      if (lane >= o2) {
        xs += a1;
        xp += a2;
        xr += a3;
      }
    }
    if (lane == 31) {
      s_stot[warp][0] = xs;
      s_stot[warp][1] = xp;
      s_stot[warp][2] = xr;
    }
  }
  __syncthreads();
  if (warp < 2) {
    const int tot_sub = s_stot[0][0] + s_stot[1][0], tot_pt = s_stot[0][1] + s_stot[1][1];
    const int tot_ring = s_stot[0][2] + s_stot[1][2];
    const int sub0 = xs - my_sub + (warp ? s_stot[0][0] : 0);
    const int pt0 = xp - my_pt + (warp ? s_stot[0][1] : 0);
    const int ring0 = xr - my_ring + (warp ? s_stot[0][2] : 0);
    const bool pt_ok = tot_pt <= kFlatPtMax;
    if (ks < nseg) {
      sg.n0 = sub0;
      sg.n1 = sub0 + my_sub;
      sg.pt0 = (pt_ok && sg.s1 > sg.s0) ? pt0 : -1;
      sg.sp_idx = (pt_ok && FUSED && (sg.ply & 1)) ? pt0 + my_pt - 1 : -1;
      sg.ring_idx = my_ring ? ring0 : -1;
      if (pt_ok) {
        for (int p = p0; p <= p1; ++p) s_ptsrc[pt0 + p - p0] = li * c.maxp + p;
        if (sg.sp_idx >= 0) s_ptsrc[sg.sp_idx] = li * c.maxp + sg.plx / c.P;
      }
      if (my_ring) s_ringsrc[ring0] = li * c.w + (sg.t + 1) % c.w;
      segs[ks] = sg;
      s_n0[ks] = sub0;
    }
    if (tid == 0) {
      s_nseg = nseg;
      s_nsub = tot_sub;
      s_npt = pt_ok ? tot_pt : 0;
      s_nring = tot_ring;
    }
  }
  __syncthreads();
  nseg = s_nseg;
  const int nsub = s_nsub;
  const bool table = nsub <= kFlatSubMax;
  // page ids and ring entries in one round trip, and meanwhile the sub-tile
  // descriptors, one thread per sub-tile: chunk i of a segment covers slots
  // [max(s0, (s0/C + i) C), min(s1, (s0/C + i + 1) C)), C the chunk size
  for (int i = tid; i < s_npt; i += kFlatThreads) s_pt[i] = c.page_table[s_ptsrc[i]];
  if (FUSED)
    for (int i = tid; i < s_nring; i += kFlatThreads) s_ring[i] = c.ring[s_ringsrc[i]];
  int4 dsc[(kFlatSubMax + kFlatThreads - 1) / kFlatThreads];
  if (table) {
#pragma unroll
    for (int e = 0; e < (kFlatSubMax + kFlatThreads - 1) / kFlatThreads; ++e) {
      const int n = tid + e * kFlatThreads;
      if (n >= nsub) break;
      int lo = 0, hi = nseg - 1;  // the segment holding sub-tile n
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_n0[mid] <= n) lo = mid; else hi = mid - 1;
      }
      const FlatSeg& gs = segs[lo];
      int slot = gs.s0, rows = 0;
      if (gs.s1 > gs.s0) {
        const int cs = gs.s0 / chunk + (n - s_n0[lo]);
        slot = max(gs.s0, cs * chunk);
        rows = min(gs.s1, cs * chunk + chunk) - slot;
      }
      const int pte = gs.pt0 >= 0 && rows > 0 ? gs.pt0 + slot / c.P - gs.s0 / c.P : -1;
      dsc[e] = make_int4(slot, rows | (lo << 8), 0, pte);
    }
  }
  __syncthreads();
  if (table) {
    // pool rows of the sub-tiles (and FP8 page scales)
#pragma unroll
    for (int e = 0; e < (kFlatSubMax + kFlatThreads - 1) / kFlatThreads; ++e) {
      const int n = tid + e * kFlatThreads;
      if (n >= nsub) break;
      int4 d = dsc[e];
      if ((d.y & 255) > 0) {
        const FlatSeg& gs = segs[d.y >> 8];
        const int page = d.w >= 0 ? s_pt[d.w] : c.page_table[(lbase + gs.bh) * c.maxp + d.x / c.P];
        d.z = page * c.P + d.x % c.P;
        if (FP8) {
          s_ks[n] = c.k_scale[page];
          s_vs[n] = c.v_scale[page];
        }
      }
      s_sub[n] = d;
    }
  }
  __syncthreads();
  // Early: the producer starts the first ring of K/V loads (this layer's
  // pages) before waiting; the aux warp waits before reading the inputs and
  // the shared counters; the consumers see only what those two publish.
  // The other warps of the CTA do not wait themselves.

  // Finish head segs[k]: LSE merge of its sources (the CTA's merged state
  // `cp` when it holds the whole head, else the partials in global scratch)
  // and, fused, the new token; output rows; append.  Threads tix of nth.
  auto finish_head = [&](int k, const float* cp, int tix, int nth) {
        const FlatSeg& sg = segs[k];
        const int bh = sg.bh, b = bh / c.Hkv, h = bh % c.Hkv;
        const long li = lbase + bh;
        const int np = sg.nparts;
        auto pslot_of = [&](int p) {
          const int cpi = U < G ? cta_of(sg.unit0 + p) : sg.first_cta + p;
          return static_cast<long>(p == 0 ? sg.first_pslot : 2 * cpi);
        };
        // online LSE merge of the sources, one lane per (row, 4 columns)
        constexpr int Q4 = D / 4;
        for (int idx = tix; idx < g * Q4; idx += nth) {
          const int r = idx / Q4, d4 = idx % Q4;
          float M = -INFINITY, L = 0.f;
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
          auto add = [&](float m, float l, float4 v) {
            if (m == -INFINITY) return;  // a source without visible keys
            if (m > M) {
              const float f = exp2f(M - m);
              a.x *= f;
              a.y *= f;
              a.z *= f;
              a.w *= f;
              L *= f;
              M = m;
            }
            const float wgt = exp2f(m - M);
            L = fmaf(wgt, l, L);
            a.x = fmaf(wgt, v.x, a.x);
            a.y = fmaf(wgt, v.y, a.y);
            a.z = fmaf(wgt, v.z, a.z);
            a.w = fmaf(wgt, v.w, a.w);
          };
          uint2 vv = make_uint2(0u, 0u);
          if (FUSED)
            vv = k < kFlatPrefetch ? *reinterpret_cast<const uint2*>(&s_kvnew[k][1][4 * d4])
                                   : *reinterpret_cast<const uint2*>(v_new + static_cast<long>(bh) * D + 4 * d4);
          if (np == 1) {
            const float* cr = cp + r * MLD;
            add(cr[D], cr[D + 1], make_float4(cr[4 * d4], cr[4 * d4 + 1], cr[4 * d4 + 2], cr[4 * d4 + 3]));
          } else {
            int p = 0;
            for (; p + 4 <= np; p += 4) {
              float4 v[4];
              float2 ml[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const long ps = pslot_of(p + u);
                v[u] = __ldcg(reinterpret_cast<const float4*>(c.part_acc + (ps * g + r) * D) + d4);
                ml[u] = __ldcg(reinterpret_cast<const float2*>(c.part_ml + (ps * g + r) * 2));
              }
#pragma unroll
              for (int u = 0; u < 4; ++u) add(ml[u].x, ml[u].y, v[u]);
            }
            for (; p < np; ++p) {
              const long ps = pslot_of(p);
              const float2 ml = __ldcg(reinterpret_cast<const float2*>(c.part_ml + (ps * g + r) * 2));
              add(ml.x, ml.y, __ldcg(reinterpret_cast<const float4*>(c.part_acc + (ps * g + r) * D) + d4));
            }
          }
          if (FUSED) {
            const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv.x));
            const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv.y));
            add(s_x[k][r], 1.0f, make_float4(v01.x, v01.y, v23.x, v23.y));
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
          uint2 pk;
          pk.x = pack_bf16(a.x * inv, a.y * inv);
          pk.y = pack_bf16(a.z * inv, a.w * inv);
          *reinterpret_cast<uint2*>(o + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g + r) * D + 4 * d4) =
              pk;
        }
        if (FUSED) {
          // append of the token at the planned slot: every CTA reading this
          // head has arrived, so its pages are no longer read in this launch
          const int flags = sg.ply, slot = sg.plx, t = sg.t, cnt = sg.cnt;
          bool okp = !(flags & 4);
          int id = -1;
          const int np_old = sg.npages;
          if (okp && (flags & 2)) {
            id = s_next_page0 + sg.grant;
            if (id >= c.pool_pages || np_old >= c.maxp) okp = false;
          } else if (okp) {
            id = sg.sp_idx >= 0 ? s_pt[sg.sp_idx] : c.page_table[li * c.maxp + slot / c.P];
          }
          int cnt_new = cnt, np_new = np_old;
          if (okp) {
            const long row = static_cast<long>(id) * c.P + slot % c.P;
            for (int e = tix; e < D / 8; e += nth) {
              const uint4* ksrc = k < kFlatPrefetch ? reinterpret_cast<const uint4*>(s_kvnew[k][0])
                                                    : reinterpret_cast<const uint4*>(k_new + static_cast<long>(bh) * D);
              const uint4* vsrc = k < kFlatPrefetch ? reinterpret_cast<const uint4*>(s_kvnew[k][1])
                                                    : reinterpret_cast<const uint4*>(v_new + static_cast<long>(bh) * D);
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.k_pool) + row * D)[e] = ksrc[e];
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.v_pool) + row * D)[e] = vsrc[e];
            }
            if (!(flags & 1)) cnt_new = cnt + 1;
            if (flags & 2) np_new += 1;
          }
          if (tix == 0) {
            if (okp) {
              if (flags & 2) {
                c.page_table[li * c.maxp + np_new - 1] = id;
                c.npages[li] = np_new;
                atomicAdd(&s_grants, 1);
              }
              const int hs = (fuse_decide || c.alpha_per != DMS_ALPHA_PER_LAYER) ? h : 0;
              const float av = s_alpha[k] == s_alpha[k] ? s_alpha[k] : __ldcg(&alpha[b * c.Hkv + hs]);
              const bool evict = shifted_mark(c, li, t, !c.disable && av > 0.0f);
              c.slot_pos[li * c.cap + slot] = t;
              c.ring[li * c.w + t % c.w] = slot | (evict ? static_cast<int>(RING_EVICT) : 0);
              if (!(flags & 1)) c.count[li] = cnt_new;
            } else {
              set_status(c.ctrl, (flags & 4) ? DMS_ST_CAPACITY : DMS_ST_POOL_EXHAUSTED);
            }
            // plan of the next append (token t + 1), with its count snapshot
            const int tn = t + 1;
            const int rn = sg.ring_idx >= 0 ? s_ring[sg.ring_idx] : 0;
            *plan_at(c, li, tn) = make_plan(rn, tn, cnt_new, np_new, c);
          }
        }
      };

  if (warp == kFlatAux) {
    // ---- aux: first what the append of each head needs, while the tiles
    // stream (the new token's scores and K/V rows, its decision logit) ------
    if (early) {
      griddep_wait();
      griddep_launch_dependents();
    }
    if (FUSED && lane == 0) s_next_page0 = c.ctrl[CTRL_NEXT_PAGE];  // read by finishes after aux_done
    __syncwarp();
    if (FUSED) {
      for (int k = 0; k < nseg; ++k) {
        const FlatSeg& sg = segs[k];
        const int bh = sg.bh, b = bh / c.Hkv, h = bh % c.Hkv;
        const __nv_bfloat16* qrow = q + (static_cast<long>(b) * c.Hq + static_cast<long>(h) * g) * D;
        const __nv_bfloat16* kn = k_new + static_cast<long>(bh) * D;
        const __nv_bfloat16* vn = v_new + static_cast<long>(bh) * D;
        float kv[D / 32];
        __nv_bfloat16 kb[D / 32], vb[D / 32];
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          kb[j] = kn[lane + 32 * j];
          vb[j] = vn[lane + 32 * j];
          kv[j] = __bfloat162float(kb[j]);
        }
        if (k < kFlatPrefetch) {
#pragma unroll
          for (int j = 0; j < D / 32; ++j) {
            s_kvnew[k][0][lane + 32 * j] = kb[j];
            s_kvnew[k][1][lane + 32 * j] = vb[j];
          }
        }
        for (int r = 0; r < g; ++r) {
          float sdot = 0.f;
#pragma unroll
          for (int j = 0; j < D / 32; ++j)
            sdot = fmaf(__bfloat162float(qrow[static_cast<long>(r) * D + lane + 32 * j]), kv[j], sdot);
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o2);
          if (lane == 0) s_x[k][r] = sdot * sl2;
        }
        float a = 0.f;
        if (sg.decide) {
          // decision logit of a head whose first unit is here (layer
          // granularity: head 0's logit for every head)
          a = decide_warp(c, da, b, c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h);
          if (lane == 0) alpha[b * c.Hkv + h] = a;
        } else if (!fuse_decide) {
          // written by the neuron pass before this launch
          a = __ldcg(&alpha[b * c.Hkv + (c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h)]);
        } else {
          a = NAN;  // computed by another CTA: read when finishing
        }
        if (lane == 0) s_alpha[k] = a;
      }
      __threadfence();  // the logits written here are visible before any hand-over
    }
    __syncwarp();
    // ---- hand-overs, in segment order: the consumers' merged state of
    // segment k arrives in cpart[k & 1].  A head held here alone is finished
    // here from it; a head shared with other CTAs leaves its partial and
    // counts its arrival, and its last arrival is queued for the consumers
    // (a merge over global partials wants more than one warp)
    bool aux_timed_out = false;
    for (int k = 0; k < nseg; ++k) {
      const int j = k & 1;
      if (!mbar_wait_bounded(&hq_full[j], (k >> 1) & 1)) aux_timed_out = true;
      const FlatSeg& sg = segs[k];
      const float* cp = cpart + j * g * MLD;
      const int bh = sg.bh;
      bool finish = sg.nparts == 1;
      if (!finish) {
        for (int idx = lane; idx < g * (D + 2); idx += 32) {
          const int r = idx / (D + 2), d = idx % (D + 2);
          if (d < D)
            c.part_acc[(static_cast<long>(sg.pslot) * g + r) * D + d] = cp[r * MLD + d];
          else
            c.part_ml[(static_cast<long>(sg.pslot) * g + r) * 2 + (d - D)] = cp[r * MLD + d];
        }
        __syncwarp();  // the lanes' partial stores precede lane 0's release
        int last = 0;
        if (lane == 0) {
          // release: this partial is visible to whoever sees the count;
          // acquire: the last arrival sees every other part's partial
          last = atom_add_acq_rel(&c.head_done[bh], 1) == sg.nparts - 1;
          if (last) c.head_done[bh] = 0;
        }
        finish = __shfl_sync(0xffffffffu, last, 0) != 0;
      }
      if (finish && sg.nparts == 1) {
        finish_head(k, cp, lane, 32);  // held here alone: sources in shared memory
      } else if (finish && lane == 0) {
        s_fin[s_nfin++] = k;  // the head's last part: finished by the consumers
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&hq_empty[j]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&aux_done);  // releases s_fin
    if (aux_timed_out && lane == 0) set_status(c.ctrl, DMS_ST_TIMEOUT);
  } else if (warp == kFlatProducer) {
    // ---- producer: one thread issues every TMA load of this CTA -----------
    if (lane == 0) {
      bool timed_out = false;
      const int mper = nst / kFlatConsumers;
      const uint64_t kv_policy = l2_evict_first_policy();
      // sub-tile n into its stage once the stage's previous use is released:
      // K and V boxes, then (issue_q) the head's query rows, one mbarrier
      // transaction for both
      auto issue_kv = [&](int n, int slot, int rows, int row0, float ks, float vs) -> unsigned char* {
        int st, use;
        flat_stage(n, mper, &st, &use);
        if (use > 0 && !mbar_wait_bounded(&empty_bar[st], (use - 1) & 1)) timed_out = true;
        FlatMeta m;
        m.slot = slot;
        m.rows = rows;
        m.ks = ks;
        m.vs = vs;
        meta[st] = m;
        unsigned char* dst = sbase + st * stride;
        const uint32_t bytes = (rows > 0 ? 2u * F::TILE : 0u) + static_cast<uint32_t>(g * D * 2);
        mbar_expect_tx(&full_bar[st], bytes);
        if (rows > 0) {
          if (FP8) {
            tma_load_2d_hint(dst, &kmap, 0, row0, &full_bar[st], kv_policy);
            tma_load_2d_hint(dst + F::TILE, &vmap, 0, row0, &full_bar[st], kv_policy);
          } else {
#pragma unroll
            for (int hf = 0; hf < F::HALVES; ++hf) {
              tma_load_2d_hint(dst + hf * kFlatRows * 128, &kmap, hf * 64, row0, &full_bar[st], kv_policy);
              tma_load_2d_hint(dst + F::TILE + hf * kFlatRows * 128, &vmap, hf * 64, row0, &full_bar[st],
                               kv_policy);
            }
          }
        }
        return dst;
      };
      auto issue_q = [&](int n, int qoff) {
        int st, use;
        flat_stage(n, mper, &st, &use);
        bulk_load(sbase + st * stride + 2 * F::TILE, q + qoff, static_cast<uint32_t>(g * D * 2), &full_bar[st]);
      };
      auto issue = [&](int n, int slot, int rows, int row0, float ks, float vs, int qoff) {
        issue_kv(n, slot, rows, row0, ks, vs);
        issue_q(n, qoff);
      };
      int n_early = 0;
      if (early && table) {
        // the first ring of K/V while the previous kernel may still run
        n_early = min(nsub, nst);
        for (int n = 0; n < n_early; ++n) {
          const int4 d = s_sub[n];
          issue_kv(n, d.x, d.y & 255, d.z, FP8 ? s_ks[n] : 1.0f, FP8 ? s_vs[n] : 1.0f);
        }
      }
      if (early) {
        griddep_wait();
        griddep_launch_dependents();
      }
      for (int n = 0; n < n_early; ++n) issue_q(n, segs[s_sub[n].y >> 8].qoff);
      if (table) {
        for (int n = n_early; n < nsub; ++n) {
          const int4 d = s_sub[n];
          issue(n, d.x, d.y & 255, d.z, FP8 ? s_ks[n] : 1.0f, FP8 ? s_vs[n] : 1.0f, segs[d.y >> 8].qoff);
        }
      } else {
        // more sub-tiles than the descriptor table holds: worked out on the way
        int n = 0;
        for (int k = 0; k < nseg; ++k) {
          const FlatSeg sg = segs[k];
          const long lh = lbase + sg.bh;
          int s = sg.s0;
          do {
            const int rows = s < sg.s1 ? min(sg.s1, (s / chunk + 1) * chunk) - s : 0;
            int row0 = 0;
            float ks = 1.0f, vs = 1.0f;
            if (rows > 0) {
              const int pi = s / c.P;
              const int page = sg.pt0 >= 0 ? s_pt[sg.pt0 + pi - sg.s0 / c.P] : c.page_table[lh * c.maxp + pi];
              row0 = page * c.P + s % c.P;
              if (FP8) {
                ks = c.k_scale[page];
                vs = c.v_scale[page];
              }
            }
            issue(n, s, rows, row0, ks, vs, sg.qoff);
            s += rows;
            ++n;
          } while (s < sg.s1);
        }
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int j = max(0, nsub - nst); j < nsub; ++j) {
        int st, use;
        flat_stage(j, mper, &st, &use);
        if (!mbar_wait_bounded(&full_bar[st], use & 1)) timed_out = true;
      }
      if (timed_out) set_status(c.ctrl, DMS_ST_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---- consumers ---------------------------------------------------------
    // TQ (g <= 8): keys as the mma M dimension (warp_tile_keys_t), else queries
    constexpr int NA = TQ ? D / 16 : NT;
    uint32_t qa[KS][4], qt[KS][2];
    float acc[NA][4];
    float mrow[2], lrow[2];
    bool timed_out = false;
    for (int k = 0; k < nseg; ++k) {
      const FlatSeg& sg = segs[k];
#pragma unroll
      for (int nt = 0; nt < NA; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      mrow[0] = mrow[1] = -INFINITY;
      lrow[0] = lrow[1] = 0.f;
      bool have_q = false;
      const int masked_slot = (FUSED && (sg.ply & 1)) ? sg.plx : -1;
      // this warp's sub-tiles of the segment: n = warp (mod 4)
      for (int n = sg.n0 + ((warp - sg.n0) % kFlatConsumers + kFlatConsumers) % kFlatConsumers; n < sg.n1;
           n += kFlatConsumers) {
        int st, use;
        flat_stage(n, nst / kFlatConsumers, &st, &use);
        const bool ok = mbar_wait_bounded(&full_bar[st], use & 1);
        if (!ok) timed_out = true;
        const FlatMeta m = meta[st];
        const unsigned char* stage = sbase + st * stride;
        if (!have_q) {
          load_q_frags<D>(reinterpret_cast<const __nv_bfloat16*>(stage + 2 * F::TILE), g, qa);
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            qt[ks][0] = qa[ks][0];
            qt[ks][1] = qa[ks][2];
          }
          have_q = true;
        }
        if (ok && m.rows > 0) {
          const int masked = masked_slot >= 0 ? masked_slot - m.slot : -1;
          // (a 32-row box is always loaded: rows past the sub-tile are pool
          // rows, finite, and masked)
          const unsigned char* kt = stage;
          const unsigned char* vt = stage + F::TILE;
          float kl2 = sl2, vs = 1.0f;
          if (FP8) {
            unsigned char* cv = conv_buf + warp * F::CONV_WARP;
            widen_fp8_rows<D, F::CROWS, kFlatRows>(stage, cv, 0);
            __syncwarp();
            kt = cv;
            vt = cv + F::CROWS * D * 2;
            kl2 = m.ks * sl2;
            vs = m.vs;
          }
          if constexpr (TQ)
            warp_tile_keys_t<D, kFlatRows, kFlatRows>(kt, vt, m.rows, masked, kl2, vs, qt, acc, mrow, lrow);
          else
            warp_tile_keys<D, kFlatRows, kFlatRows>(kt, vt, m.rows, masked, kl2, vs, qa, acc, mrow, lrow);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);
      }

      // ---- end of a segment: merge the four warps' states into cpart[k & 1]
      // (once the aux warp has released it) and hand it over -----------------
      const int j = k & 1;
      if constexpr (TQ)
        warp_state_t_to_smem<D>(merge, warp, g, acc, mrow, lrow);
      else
        warp_state_to_smem<D>(merge, warp, g, acc, mrow, lrow);
      if (k >= 2 && !mbar_wait_bounded(&hq_empty[j], ((k >> 1) - 1) & 1)) timed_out = true;
      consumers_sync();
      float* cpj = cpart + j * g * MLD;
      merge_sources<D>(merge, kFlatConsumers, g, 1.0f, [&](int r, int d, float v) { cpj[r * MLD + d] = v; });
      consumers_sync();
      if (tid == 0) mbar_arrive(&hq_full[j]);
    }
    // the heads whose last part arrived here, once every hand-over is done
    if (!mbar_wait_bounded(&aux_done, 0)) timed_out = true;
    for (int f = 0; f < s_nfin; ++f) finish_head(s_fin[f], nullptr, tid, 128);
    if (timed_out && lane == 0) set_status(c.ctrl, DMS_ST_TIMEOUT);
  }

  if (FUSED) {
    // the grid's last CTA advances the page counter and the positions (every
    // CTA's aux warp read the counter, and every head its position, before
    // this barrier)
    __syncthreads();
    if (tid == 0) s_last = count_step(c, s_grants, G, s_next_page0) ? 1 : 0;
    __syncthreads();
    if (s_last) advance_positions(c, layer, tid, kFlatThreads);
  }
}

// Launch geometry of the flat kernel, or false when the shape is outside what
// it stages in shared memory (the caller then takes the cluster kernel).
template <int D, bool FP8, bool FUSED, bool TQ>
static bool flat_geometry(const CacheView& c, int* grid, int* nst, size_t* smem) {
  using F = FlatSmem<D, FP8>;
  static int budget = -1;  // dynamic shared memory a block may take beside its static arrays
  if (budget < 0) {
    int dev = 0, optin = 0;
    cudaFuncAttributes fa{};
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, k_decode_flat<D, FP8, FUSED, TQ>) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    budget = optin - static_cast<int>(fa.sharedSizeBytes);
  }
  const int g = c.Hq / c.Hkv, BH = c.B * c.Hkv;
  const int G = std::min(c.num_sms, c.items_cap / 2);
  if (G <= 0) return false;
  // the largest unit (2048 slots) must leave every CTA at most kFlatSegMax - 2 units
  if ((BH + G - 1) / G > kFlatSegMax - 2) return false;
  const size_t fixed = F::fixed(g), stride = F::stage_stride(g);
  if (budget <= 0 || fixed + kFlatConsumers * stride > static_cast<size_t>(budget)) return false;
  // a whole number of stages per consumer warp
  const int n = static_cast<int>(std::min<size_t>(kFlatMaxStages, (budget - fixed) / stride)) / kFlatConsumers *
                kFlatConsumers;
  if (n < kFlatConsumers) return false;
  // the partition scratch (7 ints per head) lives in the stage ring
  if (static_cast<size_t>(7 * BH + 8) * sizeof(int) > n * stride) return false;
  *grid = G;
  *nst = n;
  *smem = fixed + n * stride;
  return true;
}

template <int D, bool FP8, bool FUSED, bool TQ>
static cudaError_t launch_flat_t(const CacheView& c, int layer, const void* q, void* o, const void* k, const void* v,
                                 float* alpha, const DecideArgs* da, const CUtensorMap* kmap, const CUtensorMap* vmap,
                                 cudaStream_t s, bool early, bool* taken) {
  int grid = 0, nst = 0;
  size_t smem = 0;
  *taken = (reinterpret_cast<uintptr_t>(q) & 15) == 0 && flat_geometry<D, FP8, FUSED, TQ>(c, &grid, &nst, &smem);
  if (!*taken) return cudaSuccess;
  auto kern = k_decode_flat<D, FP8, FUSED, TQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  DecideArgs none{};
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kFlatThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, c, layer, early ? 1 : 0, static_cast<const __nv_bfloat16*>(q),
                            static_cast<__nv_bfloat16*>(o), nst, static_cast<const __nv_bfloat16*>(k),
                            static_cast<const __nv_bfloat16*>(v), alpha, da ? *da : none, da ? 1 : 0, *kmap, *vmap);
}

// One instantiation per (head dim, page type, fused step, key-major tiles).
template <bool FP8, bool FUSED>
static cudaError_t launch_flat_dt(const CacheView& c, int layer, const void* q, void* o, const void* k, const void* v,
                                  float* alpha, const DecideArgs* da, const CUtensorMap* kmap, const CUtensorMap* vmap,
                                  cudaStream_t s, bool early, bool* taken) {
  const bool tq = c.Hq / c.Hkv <= 8;
  if (c.D == 64)
    return tq ? launch_flat_t<64, FP8, FUSED, true>(c, layer, q, o, k, v, alpha, da, kmap, vmap, s, early, taken)
              : launch_flat_t<64, FP8, FUSED, false>(c, layer, q, o, k, v, alpha, da, kmap, vmap, s, early, taken);
  return tq ? launch_flat_t<128, FP8, FUSED, true>(c, layer, q, o, k, v, alpha, da, kmap, vmap, s, early, taken)
            : launch_flat_t<128, FP8, FUSED, false>(c, layer, q, o, k, v, alpha, da, kmap, vmap, s, early, taken);
}

cudaError_t launch_decode_flat(const CacheView& c, int layer, const void* q, void* o, bool fused, const void* k,
                               const void* v, float* alpha, const DecideArgs* fused_decide, const CUtensorMap* kmap,
                               const CUtensorMap* vmap, cudaStream_t s, bool early, bool* taken) {
  *taken = false;
  if (!kmap || !vmap || c.kv_dtype == DMS_F32) return cudaErrorInvalidValue;
  if (fused) {
    if (c.kv_dtype != DMS_BF16) return cudaErrorInvalidValue;
    return launch_flat_dt<false, true>(c, layer, q, o, k, v, alpha, fused_decide, kmap, vmap, s, early, taken);
  }
  if (c.kv_dtype == DMS_FP8_E4M3)
    return launch_flat_dt<true, false>(c, layer, q, o, k, v, alpha, nullptr, kmap, vmap, s, early, taken);
  return launch_flat_dt<false, false>(c, layer, q, o, k, v, alpha, nullptr, kmap, vmap, s, early, taken);
}

}  // namespace dms

