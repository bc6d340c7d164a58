// Decode attention with one thread-block cluster per KV head, and the fused
// decode step built on it.
//
// A cluster of `cs` CTAs (cs a power of two <= 8, chosen so the grid fits the
// SMs at the CTAs per SM its shared memory allows, at most two) covers one
// (b, h): CTA r attends a contiguous range of the head's retained slots, cut
// at multiples of 32 slots (16 when the page size is not a multiple of 32) so
// no sub-tile crosses a page.  Sub-tile n belongs to warp n mod 4, which
// issues its TMA loads into stages of its own, waits on them and runs the
// whole online-softmax update of its keys with the g query heads as the M
// dimension of mma.sync tiles: the four warps stream independently, with no
// block barrier between sub-tiles.  Each CTA merges its warps into one partial (acc, running
// max, running sum, log2 domain) and writes it with st.async into the shared
// memory of the cluster's last rank (the owner), completing bytes on an
// mbarrier there; the owner, whose share of the slots is the smallest, merges
// the cs partials from its own shared memory and writes the head's output
// rows ([FastDMS], attention scoring: split-K grouped compact decode
// attention over variable-length per-head live spans -- here the split never
// leaves the chip).  The other ranks leave as soon as their partial is sent.
//
// FUSED (bf16 pages): the whole decode step in one launch.  The attention runs
// over the slots as they were before this step's append, with the slot this
// token reuses masked out and the new token's key/value taken from the input
// as one more key of rank 0 -- the same visible set as after the append.  Rank
// 0 (the owner) then appends the token at the slot fixed by the plan of the previous step
// ([DMS-Qwen3], inference mode: a token overwrites the slot of the token
// leaving the window when that one was marked, else takes the next slot; a new
// page when that slot starts one), updates the head's count and writes the
// plan of the next append.  New pages are numbered from the page counter as
// read at the start plus the head's rank among the heads needing one, i.e. in
// (b, h) row-major order; the grid's last CTA advances the counter and the
// positions.
#include "decode_common.cuh"

namespace dms {


constexpr int kMaxCluster = 16;  // shared-memory staging bound
constexpr int kPickCluster = 8;  // largest cluster launched: every cluster of the grid co-resident

__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Slots per warp sub-tile: one TMA box of that many rows per K / V column
// half (32 rows; 64-row FP8 boxes of 64-byte rows measured slower).
__host__ __device__ constexpr int cluster_rows(int D, bool FP8) { return (void)D, (void)FP8, 32; }

template <int D, bool FP8, bool TQ>
struct ClusterSmem {
  static constexpr int ROWS = cluster_rows(D, FP8);
  static constexpr int TILE = FP8 ? ROWS * D : ROWS * D * 2;      // K (or V) of one sub-tile, as loaded
  static constexpr int STAGE = 2 * TILE;                           // K then V (a multiple of 1024 bytes)
  static constexpr int MPER = D == 64 ? 4 : 2;                     // stages per warp (at most)
  static constexpr int NST = 4 * MPER;
  // widened FP8 codes per warp: V (to f16) with key-major tiles, else K and V (to bf16)
  static constexpr int CONV_WARP = FP8 ? (TQ ? 1 : 2) * ROWS * D * 2 : 0;
  static constexpr int MLD = D + 2;
  static constexpr int IMLD = D + 4;  // inbox row: D values, max, sum, 2 pad (16-byte rows)
  // floats of the merge buffer [4 warps][g][MLD], rounded up so the inbox
  // after it starts on 16 bytes
  __host__ __device__ static int merge_floats(int g) { return (4 * g * MLD + 3) / 4 * 4; }
  // stages, conversion tiles, merge buffer, the owner's inbox [cs][g][IMLD]
  static size_t bytes(int g, int cs, int mper) {
    return 1024 + 4 * mper * STAGE + 4 * CONV_WARP + (merge_floats(g) + cs * g * IMLD) * sizeof(float);
  }
};

struct SubMeta {
  int slot;  // first slot of the sub-tile
  int rows;  // slots in the sub-tile (<= 64, inside one page)
  int page;  // page id
};

template <int D, bool FP8, bool FUSED, bool TQ>
__global__ void __launch_bounds__(kThreads, 1) k_decode_cluster(CacheView c, int layer, int nl, int early,
                                                            const __nv_bfloat16* q, __nv_bfloat16* o, int cs,
                                                            int mper,
                                                            const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                                            float* alpha, DecideArgs da, int fuse_decide,
                                                            const __grid_constant__ CUtensorMap kmap,
                                                            const __grid_constant__ CUtensorMap vmap) {
  using S = ClusterSmem<D, FP8, TQ>;
  constexpr int KS = D / 16, NT = D / 8, MLD = D + 2, IMLD = S::IMLD;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sbase =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* stage_buf = sbase;                              // [4 mper] stages; warp w owns w, w + 4, ...
  unsigned char* conv_buf = sbase + 4 * mper * S::STAGE;         // FP8: [4 warps] widened K, V
  const int g = c.Hq / c.Hkv;
  float* merge = reinterpret_cast<float*>(conv_buf + 4 * S::CONV_WARP);  // [4 warps][g][MLD]
  float* inbox = merge + S::merge_floats(g);  // [cs][g][IMLD] partials, on the owner (16-byte aligned)
  __shared__ uint64_t full_bar[S::NST];
  __shared__ uint64_t inbox_bar;  // the owner: every rank's partial has landed
  __shared__ SubMeta meta[S::NST];
  __shared__ int s_ring_next;
  __shared__ float s_fred[8], s_alpha;
  __shared__ int s_app_ok, s_app_id;  // append-first step: the owner's append succeeded, its page
  __shared__ float s_app_sc[2];       // ... and the page's K and V scales after it
  __shared__ __align__(16) __nv_bfloat16 s_knew[D], s_vnew[D];
  __shared__ float s_xs[16];  // the new token's scores (log2 domain), owner of a bf16 step
  constexpr int kPtCache = 256;  // page-table entries of the head kept in shared memory
  __shared__ int s_pt[kPtCache];
  __shared__ float s_ksc[FP8 ? kPtCache : 1], s_vsc[FP8 ? kPtCache : 1];  // FP8 page scales

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // head vh of the launch: (layer + lrel, b, h); the inputs of a multi-layer
  // launch hold its layers back to back, so their row is bb = lrel * B + b
  const int vh = blockIdx.x / cs, BH = c.B * c.Hkv;
  const int lrel = vh / BH, bh = vh % BH;
  const int rank = static_cast<int>(cluster_rank());
  const int owner = cs - 1;  // the rank that appends: its slice of the slots is the shortest
  const int b = bh / c.Hkv, h = bh % c.Hkv, bb = vh / c.Hkv;
  const long li = static_cast<long>(layer) * BH + vh;
  // Programmatic dependent launch.  With `early` (the previous launch of this
  // library on the stream was for another layer or cache) this layer's state
  // is read and the first tiles are requested before waiting for the previous
  // kernel: only that kernel may still run (each kernel lets its dependents
  // start only once its own wait has returned), and it does not write this
  // state.  The page counter, the inputs and the outputs are touched only
  // after the wait.
  if (tid == 32) {
    // the pool's tensor maps, fetched while the head's state is read
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
  }
  if (!early) {
    griddep_wait();
    griddep_launch_dependents();
  }
  if (tid == 0) {
    for (int i = 0; i < 4 * mper; ++i) mbar_init(&full_bar[i], 1);
    mbar_init(&inbox_bar, 1);
    fence_mbar_init();
  }
  // state of this head (stable during the launch: only rank 0 of this head's
  // cluster writes it, after the cluster barrier; the position and the page
  // counter only change in the grid's last CTA)
  // the head's page-table row is fetched together with the count (no dependent round trip)
  for (int i = tid; i < min(c.maxp, kPtCache); i += kThreads) s_pt[i] = c.page_table[li * c.maxp + i];
  const int cnt = c.count[li];
  const int t = FUSED ? c.pos[layer * c.B + bb] : 0;
  // both plan buffers in the same round trip as the position that picks one
  const int4 pl0 = FUSED ? *plan_at(c, li, 0) : make_int4(0, 0, 0, 0);
  const int4 pl1 = FUSED ? *plan_at(c, li, 1) : make_int4(0, 0, 0, 0);
  const int4 pl = (t & 1) ? pl1 : pl0;
  // FP8 pages (fused step): the owner appends the token first (the page's
  // rows are re-encoded when its scale grows) and the attention reads it from
  // its page with the rest.  The visible slots are those after the append,
  // assumed to succeed (only the owner's range depends on the outcome: a
  // failed append can only drop the last slot), and page pa, which the append
  // writes, is read only after the owner's cluster arrive.  bf16 pages: the
  // attention covers the slots before the append, without the slot the
  // token reuses, and takes the token from the input.
  constexpr bool kAppendFirst = FUSED && FP8;
  const int cnt_vis = (kAppendFirst && !(pl.y & 5)) ? cnt + 1 : cnt;
  const int pa = (kAppendFirst && !(pl.y & 4)) ? pl.x / c.P : -1;
  const int masked_slot = (FUSED && !kAppendFirst && (pl.y & 1)) ? pl.x : -1;
  // The decision logit of the new token: with cs >= 4, rank 0 computes it
  // before attending a reduced share (it sends the logit with its partial),
  // so it is off the path of the other ranks; with a smaller cluster the
  // owner computes it before streaming.
  const bool rank0_decides = FUSED && fuse_decide && cs >= 4;
  const bool owner_decides = FUSED && fuse_decide && cs < 4;
  // the streaming ranks before the owner take `per` slots each, the owner
  // the rest: half a share (it merges the partials and appends), a quarter
  // share when it also computes the decision logit; rank 0 computing the
  // logit takes no slots of a short head and half a share of a long one
  // (at least 512 slots per rank), which outlasts the logit
  const int r0 = rank0_decides ? 1 : 0;  // first rank with a full share
  const int oq = owner_decides ? 1 : 2;
  const int q0 = rank0_decides && cnt_vis >= 512 * (cs - 1) ? 2 : 0;  // rank 0's share, in quarters
  const int nfull = cs - 1 - r0;
  const int per_q = 4 * nfull + q0 + oq;
  const int per = nfull == 0 ? 0 : ((4 * cnt_vis + per_q - 1) / per_q + (q0 ? 31 : 15)) / (q0 ? 32 : 16) * (q0 ? 32 : 16);
  const int r0end = q0 ? min(cnt_vis, per / 2) : 0;  // rank 0's slots [0, r0end)
  const int s_begin = rank < r0 ? 0 : min(cnt_vis, r0end + (rank - r0) * per);
  int s_end = rank < r0 ? r0end : rank == owner ? cnt_vis : min(cnt_vis, s_begin + per);
  __syncthreads();
  // this CTA's barriers are initialised (waited before the first remote
  // store); the owner of an append-first step arrives after its append
  if (!kAppendFirst || rank != owner) cluster_arrive_relaxed();

  // sub-tile n of this CTA: slots [max(s_begin, (first + n) C), min(s_end, (first + n + 1) C)),
  // inside one page (C divides P); warp n % 4 takes it into stage
  // n % 4 + 4 ((n / 4) mod mper), issued by the warp's lane 0
  constexpr int kCRows = S::ROWS;
  const int chunk = c.P % kCRows == 0 ? kCRows : c.P % 32 == 0 ? 32 : 16;
  const int first = s_begin / chunk;
  int nsub = s_end > s_begin ? (s_end - 1) / chunk - first + 1 : 0;
  // the pages are read once per step: first to leave L2, so that the small
  // per-step tensors (state, query and new rows, adapter rows) stay there
  const uint64_t kv_policy = l2_evict_first_policy();
  auto issue = [&](int n) {
    const int st = warp + 4 * ((n >> 2) % mper);
    const int slot = max(s_begin, (first + n) * chunk);
    const int rows = min(s_end, (first + n + 1) * chunk) - slot;
    const int pi = slot / c.P;
    const int page = pi < kPtCache ? s_pt[pi] : c.page_table[li * c.maxp + pi];
    meta[st].slot = slot;
    meta[st].rows = rows;
    meta[st].page = page;
    (void)rows;
    issue_tile<D, FP8, kCRows>(stage_buf + st * S::STAGE, &kmap, &vmap, page * c.P + slot % c.P, &full_bar[st],
                               kv_policy);
  };
  // this warp's first stages (those before page pa of an append-first step)
  int n_init = 0;
  if (lane == 0)
    for (int n = warp; n < nsub && n < 4 * mper; n += 4) {
      if (kAppendFirst && max(s_begin, (first + n) * chunk) / c.P == pa) break;
      issue(n);
      ++n_init;
    }
  n_init = __shfl_sync(0xffffffffu, n_init, 0);
  // the scales of this CTA's pages (FP8), requested while the first tiles
  // are in flight and stored before the streaming starts (the page an
  // append-first step writes comes from the append)
  const int sc_pf = s_begin / c.P, sc_pe = (FP8 && nsub) ? min((s_end - 1) / c.P, kPtCache - 1) : sc_pf - 1;
  const int sc_pi = sc_pf + tid;
  float sc_k = 0.f, sc_v = 0.f;
  if (FP8 && sc_pi <= sc_pe && sc_pi != pa) {
    sc_k = c.k_scale[s_pt[sc_pi]];
    sc_v = c.v_scale[s_pt[sc_pi]];
  }

  // append-first owner: what the append needs from this layer's state, before
  // the wait: this head's rank among the heads needing a new page, or the
  // page the token goes to and its scales (a new page's are 0)
  int app_rank = 0, app_page = -1;
  float app_ks = 0.f, app_vs = 0.f;
  if (kAppendFirst && rank == owner && pa >= 0) {
    if (pl.y & 2) {
      if (warp == 0) {
        int n_before = 0;
        for (int i = lane; i < vh; i += 32)
          n_before += (plan_at(c, static_cast<long>(layer) * BH + i, t)->y & 2) ? 1 : 0;
        app_rank = __reduce_add_sync(0xffffffffu, n_before);
      }
    } else {
      app_page = pa < kPtCache ? s_pt[pa] : c.page_table[li * c.maxp + pa];
      app_ks = c.k_scale[app_page];
      app_vs = c.v_scale[app_page];
    }
  }
  if (early) {
    griddep_wait();
    griddep_launch_dependents();
  }
  const int next_page0 = FUSED ? c.ctrl[CTRL_NEXT_PAGE] : 0;
  // this layer's adapter (hidden rows of the layer, its weights and offsets);
  // decision logit of the new token (layer granularity: head 0's)
  const int dsrc = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
  DecideArgs dl = da;
  if (FUSED && lrel > 0 && fuse_decide) {
    dl.hidden = static_cast<const __nv_bfloat16*>(da.hidden) + static_cast<long>(lrel) * c.B * c.hidden;
    dl.gamma = static_cast<const __nv_bfloat16*>(da.gamma) + lrel * da.gamma_lstride;
    dl.W = static_cast<const __nv_bfloat16*>(da.W) + lrel * da.w_lstride;
    if (da.bias) dl.bias = static_cast<const __nv_bfloat16*>(da.bias) + lrel * da.bias_lstride;
    dl.offset = da.offset + lrel * da.offset_lstride;
  }
  // Everything read after the wait, in one round trip while the first tiles
  // are in flight: the query rows, on the owner the new key/value row and the
  // ring entry of t + 1 (held in registers until the merge), and on the CTA
  // that computes the decision logit its operands.
  constexpr int kDV = 4;  // 16-byte vectors per thread of the decision logit's rows
  const bool decides = (rank0_decides && rank == 0) || (owner_decides && rank == owner);
  const bool one_trip = c.hidden <= kThreads * kDV * 8;
  DecideLoads<kDV> dq;
  if (decides && one_trip) decide_issue<kDV>(c, dl, b, dsrc, dq);
  // (FP8 pages with g <= 8: f16 fragments in the K fragments' k order)
  constexpr bool kF16 = FP8 && TQ;
  uint32_t qa[kF16 ? 1 : KS][4], qh[kF16 ? KS : 1][2];
  const __nv_bfloat16* qb = q + (static_cast<long>(bb) * c.Hq + static_cast<long>(h) * g) * D;
  if constexpr (kF16)
    load_q_frags_fp8<D>(qb, g, qh);
  else
    load_q_frags<D>(qb, g, qa);
  uint4 kn = make_uint4(0, 0, 0, 0), vn = kn;
  int ring_next = 0;
  if (FUSED && rank == owner) {
    if (!kAppendFirst && tid < D / 8) {
      kn = reinterpret_cast<const uint4*>(k_new + static_cast<long>(vh) * D)[tid];
      vn = reinterpret_cast<const uint4*>(v_new + static_cast<long>(vh) * D)[tid];
    }
    if (tid == 32 && t + 1 >= c.w) ring_next = c.ring[li * c.w + (t + 1) % c.w];
  }
  if (decides) {
    const float a = one_trip ? decide_reduce<kDV>(c, dq, s_fred) : decide_cta<4>(c, dl, b, dsrc, s_fred);
    if (tid == 0) {
      s_alpha = a;
      alpha[bb * c.Hkv + h] = a;
    }
  }
  if constexpr (kAppendFirst) {
    if (rank == owner) {
      // the append: page id (a new page is numbered from the counter by this
      // head's rank among the heads needing one), then the K and V codes
      const int flags = pl.y, slot = pl.x;
      bool ok = !(flags & 4);
      int id = app_page;
      if (ok && (flags & 2)) {
        if (warp == 0 && lane == 0) s_app_id = next_page0 + app_rank;
        __syncthreads();
        id = s_app_id;
        if (id >= c.pool_pages || pl.w >= c.maxp) ok = false;
      }
      float2 sc = make_float2(0.f, 0.f);
      if (ok) {
        const int rows = min(c.P, cnt_vis - pa * c.P);  // rows in use in the page after the append
        const __nv_bfloat16* kr = k_new + static_cast<long>(vh) * D;
        const __nv_bfloat16* vr = v_new + static_cast<long>(vh) * D;
        const float kx = tid < D ? __bfloat162float(kr[tid]) : 0.f, vx = tid < D ? __bfloat162float(vr[tid]) : 0.f;
        const long pbytes = static_cast<long>(c.P) * D;
        sc = fp8_append_kv(kx, vx, static_cast<uint8_t*>(c.k_pool) + id * pbytes,
                           static_cast<uint8_t*>(c.v_pool) + id * pbytes, c.k_scale + id, c.v_scale + id, app_ks,
                           app_vs, slot % c.P, rows, D, s_fred);
        if ((flags & 2) && tid == 0) c.page_table[li * c.maxp + pa] = id;  // read by ranks past kPtCache pages
      } else if (!(flags & 1)) {
        // the token has no slot: the owner's range ends before it
        s_end = cnt;
        nsub = s_end > s_begin ? (s_end - 1) / chunk - first + 1 : 0;
      }
      if (tid == 0) {
        // the outcome, read by the other ranks after the barrier
        s_app_ok = ok ? 1 : 0;
        s_app_id = id;
        s_app_sc[0] = sc.x;
        s_app_sc[1] = sc.y;
        if (pa >= 0 && pa < kPtCache) {
          s_pt[pa] = ok ? id : -1;
          s_ksc[pa] = sc.x;
          s_vsc[pa] = sc.y;
        }
      }
      fence_proxy_async_global();  // the codes, before the TMA loads that follow the barrier
      __syncthreads();
      cluster_arrive_release();
    }
    cluster_wait();
    if (rank != owner) {
      // the append's outcome from the owner's shared memory: the page's id
      // and scales (pages past the cached table read them from global memory)
      if (tid == 0) {
        const int ok = __float_as_int(ld_dsmem(dsmem_addr(&s_app_ok, owner)));
        const int id = __float_as_int(ld_dsmem(dsmem_addr(&s_app_id, owner)));
        const float ks = ld_dsmem(dsmem_addr(&s_app_sc[0], owner)), vs = ld_dsmem(dsmem_addr(&s_app_sc[1], owner));
        s_app_ok = ok;
        if (pa >= 0 && pa < kPtCache) {
          s_pt[pa] = ok ? id : -1;
          s_ksc[pa] = ks;
          s_vsc[pa] = vs;
        }
      }
      __syncthreads();
      if (!s_app_ok && !(pl.y & 1)) {
        // the token has no slot
        s_end = min(s_end, cnt);
        nsub = s_end > s_begin ? (s_end - 1) / chunk - first + 1 : 0;
      }
    }
    // the rest of this warp's first stages
    if (lane == 0)
      for (int n = warp + 4 * n_init; n < nsub && n < 4 * mper; n += 4) issue(n);
  }
  if (FP8) {
    if (sc_pi <= sc_pe && sc_pi != pa) {
      s_ksc[sc_pi] = sc_k;
      s_vsc[sc_pi] = sc_v;
    }
    for (int pi = sc_pf + kThreads + tid; pi <= sc_pe; pi += kThreads) {
      if (pi == pa) continue;
      s_ksc[pi] = c.k_scale[s_pt[pi]];
      s_vsc[pi] = c.v_scale[s_pt[pi]];
    }
  }
  // TQ (g <= 8): keys as the mma M dimension (warp_tile_keys_t), else queries
  constexpr int NA = TQ ? D / 16 : NT;
  float acc[NA][4];
#pragma unroll
  for (int nt = 0; nt < NA; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  uint32_t qt[kF16 ? 1 : KS][2];
  if constexpr (!kF16) {
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qt[ks][0] = qa[ks][0];
      qt[ks][1] = qa[ks][2];
    }
  }
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  if (FUSED && !kAppendFirst && rank == owner) {
    // the new token's rows and ring entry for the merge and the append, and
    // (warp 0, once its query rows and the new key have landed) its scores
    // q_r . k_new from the query fragments: lane holds columns
    // 2 (lane % 4) + {0, 1, 8, 9} of every 16 of rows lane / 4 and lane / 4 + 8
    if (tid < D / 8) {
      reinterpret_cast<uint4*>(s_knew)[tid] = kn;
      reinterpret_cast<uint4*>(s_vnew)[tid] = vn;
    }
    if (warp == 0) {
      __syncwarp();
      const int ra = lane >> 2, rb = ra + 8;
      float sa = 0.f, sb = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int col = ks * 16 + 2 * (lane & 3);
        const float2 k0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&s_knew[col]));
        const float2 k1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&s_knew[col + 8]));
        const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qa[ks][0]));
        const float2 b0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qa[ks][1]));
        const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qa[ks][2]));
        const float2 b1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qa[ks][3]));
        sa = fmaf(a0.x, k0.x, fmaf(a0.y, k0.y, fmaf(a1.x, k1.x, fmaf(a1.y, k1.y, sa))));
        sb = fmaf(b0.x, k0.x, fmaf(b0.y, k0.y, fmaf(b1.x, k1.x, fmaf(b1.y, k1.y, sb))));
      }
#pragma unroll
      for (int o2 = 1; o2 < 4; o2 <<= 1) {
        sa += __shfl_xor_sync(0xffffffffu, sa, o2);
        sb += __shfl_xor_sync(0xffffffffu, sb, o2);
      }
      if ((lane & 3) == 0) {
        if (ra < g) s_xs[ra] = sa * sl2;
        if (rb < g) s_xs[rb] = sb * sl2;
      }
    }
  }
  if (FUSED && rank == owner && tid == 32) s_ring_next = ring_next;  // read by the append after the merge
  if (FP8) __syncthreads();  // page scales staged
  {
    // this warp's sub-tiles n = warp, warp + 4, ...: local index j, stage
    // use j / mper; the refill of a stage follows the warp's own reads of it
    unsigned char* conv = conv_buf + warp * S::CONV_WARP;
    const int nmine = nsub > warp ? (nsub - warp + 3) / 4 : 0;
    int j = 0;
    bool timed_out = false;
    for (; j < nmine; ++j) {
      const int n = warp + 4 * j, st = warp + 4 * (j % mper);
      __syncwarp();
      if (!mbar_wait_bounded(&full_bar[st], (j / mper) & 1)) {
        timed_out = true;
        break;
      }
      const SubMeta m = meta[st];
      const unsigned char* kt = stage_buf + st * S::STAGE;
      const int masked = masked_slot >= 0 ? masked_slot - m.slot : -1;
      float ks = 1.0f, vs = 1.0f;
      if (FP8) {
        const int pi = m.slot / c.P;
        ks = pi < kPtCache ? s_ksc[pi] : c.k_scale[m.page];
        vs = pi < kPtCache ? s_vsc[pi] : c.v_scale[m.page];
      }
      // (a sub-tile of at most 16 slots: the tiles of 16 keys)
      if constexpr (kF16) {
        // K straight from the FP8 rows, V widened to f16
        widen_fp8_tile<D, kCRows, true>(kt + S::TILE, conv);
        __syncwarp();
        if (kCRows > 32 && m.rows > 32)
          warp_tile_keys_fp8<D, kCRows, kCRows>(kt, conv, m.rows, masked, ks * sl2, vs, qh, acc, mrow, lrow);
        else if (m.rows > 16)
          warp_tile_keys_fp8<D, 32, kCRows>(kt, conv, m.rows, masked, ks * sl2, vs, qh, acc, mrow, lrow);
        else
          warp_tile_keys_fp8<D, 16, kCRows>(kt, conv, m.rows, masked, ks * sl2, vs, qh, acc, mrow, lrow);
      } else {
        if (FP8) {
          // K and V widened to bf16
          widen_fp8_tile<D, kCRows, false>(kt, conv);
          widen_fp8_tile<D, kCRows, false>(kt + S::TILE, conv + kCRows * D * 2);
          __syncwarp();
          kt = conv;
        }
        const unsigned char* vt = kt + (FP8 ? kCRows * D * 2 : S::TILE);
        const float kl2 = FP8 ? ks * sl2 : sl2;
        if constexpr (TQ) {
          if (kCRows > 32 && m.rows > 32)
            warp_tile_keys_t<D, kCRows, kCRows>(kt, vt, m.rows, masked, kl2, vs, qt, acc, mrow, lrow);
          else if (m.rows > 16)
            warp_tile_keys_t<D, 32, kCRows>(kt, vt, m.rows, masked, kl2, vs, qt, acc, mrow, lrow);
          else
            warp_tile_keys_t<D, 16, kCRows>(kt, vt, m.rows, masked, kl2, vs, qt, acc, mrow, lrow);
        } else {
          if (kCRows > 32 && m.rows > 32)
            warp_tile_keys<D, kCRows, kCRows>(kt, vt, m.rows, masked, kl2, vs, qa, acc, mrow, lrow);
          else if (m.rows > 16)
            warp_tile_keys<D, 32, kCRows>(kt, vt, m.rows, masked, kl2, vs, qa, acc, mrow, lrow);
          else
            warp_tile_keys<D, 16, kCRows>(kt, vt, m.rows, masked, kl2, vs, qa, acc, mrow, lrow);
        }
      }
      __syncwarp();
      if (lane == 0 && n + 4 * mper < nsub) {
        fence_proxy_async();  // this warp's reads of the stage before the copy that refills it
        issue(n + 4 * mper);
      }
    }
    if (timed_out) {
      // the copies of this warp still in flight land before the CTA exits
      for (int jj = j; jj < min(nmine, j + mper); ++jj)
        mbar_wait_bounded(&full_bar[warp + 4 * (jj % mper)], (jj / mper) & 1);
      if (lane == 0) set_status(c.ctrl, DMS_ST_TIMEOUT);
    }
  }

  // merge the warps (and, for the owner of a fused step, the new token) into
  // this CTA's partial, written into slot `rank` of the owner's inbox
  if constexpr (TQ)
    warp_state_t_to_smem<D>(merge, warp, g, acc, mrow, lrow);
  else
    warp_state_to_smem<D>(merge, warp, g, acc, mrow, lrow);
  __syncthreads();
  if (!kAppendFirst) cluster_wait();  // every CTA's barriers are initialised
  // This CTA's partial, written into slot `rank` of the owner's inbox
  // (st.async to another rank): per row the four warps' states and, for the
  // owner of a bf16 step, the new token (score q_r . k_new, weight 1, value
  // v_new) merged with weights 2^(m_s - M); each thread takes four values of
  // one row and works out that row's weights, and the thread of the row's
  // first four also sends (M, L) -- row 0 with rank 0's decision logit.
  const bool xsrc = FUSED && !kAppendFirst && rank == owner;
  const uint32_t dst = dsmem_addr(inbox + rank * g * IMLD, owner), rbar = dsmem_addr(&inbox_bar, owner);
  for (int e4 = tid; e4 < g * (D / 4); e4 += kThreads) {
    const int r = e4 / (D / 4), d = 4 * (e4 % (D / 4));
    float ms[4], M = xsrc ? s_xs[r] : -INFINITY;
#pragma unroll
    for (int sv = 0; sv < 4; ++sv) {
      ms[sv] = merge[(sv * g + r) * MLD + D];
      M = fmaxf(M, ms[sv]);
    }
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int sv = 0; sv < 4; ++sv) {
      const float wgt = exp2f(ms[sv] - Mu);
      const float* src = merge + (sv * g + r) * MLD;
      L = fmaf(wgt, src[D + 1], L);
      v.x = fmaf(wgt, src[d], v.x);
      v.y = fmaf(wgt, src[d + 1], v.y);
      v.z = fmaf(wgt, src[d + 2], v.z);
      v.w = fmaf(wgt, src[d + 3], v.w);
    }
    if (xsrc) {
      const float wgt = exp2f(s_xs[r] - Mu);
      L += wgt;
      const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&s_vnew[d]));
      const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&s_vnew[d + 2]));
      v.x = fmaf(wgt, v01.x, v.x);
      v.y = fmaf(wgt, v01.y, v.y);
      v.z = fmaf(wgt, v23.x, v.z);
      v.w = fmaf(wgt, v23.y, v.w);
    }
    const float dlog = r == 0 && rank0_decides && rank == 0 ? s_alpha : 0.f;
    if (rank != owner) {
      st_async_v4(dst + 4u * static_cast<uint32_t>(r * IMLD + d), v, rbar);
      if (d == 0) {
        if (r == 0)
          st_async_v4(dst + 4u * static_cast<uint32_t>(D), make_float4(M, L, dlog, 0.f), rbar);
        else
          st_async_v2(dst + 4u * static_cast<uint32_t>(r * IMLD + D), M, L, rbar);
      }
    } else {
      float* row = inbox + (owner * g + r) * IMLD;
      *reinterpret_cast<float4*>(row + d) = v;
      if (d == 0) {
        row[D] = M;
        row[D + 1] = L;
        if (r == 0) {
          row[D + 2] = dlog;
          row[D + 3] = 0.f;
        }
      }
    }
  }
  if (rank != owner) {
    return;  // nothing reads this CTA's shared memory
  }
  if (tid == 0) mbar_expect_tx(&inbox_bar, static_cast<uint32_t>((cs - 1) * (g * (D + 2) * 4 + 8)));
  bool landed = cs == 1 || mbar_wait_bounded(&inbox_bar, 0);
  landed = __syncthreads_and(landed);  // (one answer for the block); the owner's own partial is in place too
  if (!landed && tid == 0) set_status(c.ctrl, DMS_ST_TIMEOUT);

  if (FUSED && warp == 3) {
    // Warp 3 appends this head's token at the planned slot (every CTA of the
    // cluster has finished reading the pages: their partials have landed) and
    // counts the step, while warps 0-2 merge the output.
    const int flags = pl.y, slot = pl.x;
    int id = -1;
    bool ok = !(flags & 4);
    if (kAppendFirst) {
      // done before the attention
      ok = s_app_ok != 0;
      id = s_app_id;
    } else if (ok && (flags & 2)) {
      // a new page: numbered by this head's rank among the heads that need one
      int n_before = 0;
      for (int i = lane; i < vh; i += 32)
        n_before += (plan_at(c, static_cast<long>(layer) * BH + i, t)->y & 2) ? 1 : 0;
      n_before = __reduce_add_sync(0xffffffffu, n_before);
      id = next_page0 + n_before;
      if (id >= c.pool_pages || pl.w >= c.maxp) ok = false;
    } else if (ok) {
      const int pi = slot / c.P;
      id = pi < kPtCache ? s_pt[pi] : c.page_table[li * c.maxp + pi];
    }
    int cnt_new = cnt, np_new = pl.w;  // pages before the append (plan snapshot)
    if (ok) {
      const long row = static_cast<long>(id) * c.P + slot % c.P;
      if (!kAppendFirst && lane < D / 8) {
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.k_pool) + row * D)[lane] =
            reinterpret_cast<const uint4*>(s_knew)[lane];
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c.v_pool) + row * D)[lane] =
            reinterpret_cast<const uint4*>(s_vnew)[lane];
      }
      if (!(flags & 1)) cnt_new = cnt + 1;
      if (flags & 2) np_new += 1;
      if (lane == 0) {
        if (flags & 2) {
          c.page_table[li * c.maxp + np_new - 1] = id;
          c.npages[li] = np_new;
        }
        const int hs = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
        const float a = rank0_decides ? inbox[D + 2]  // rank 0's row 0
                        : owner_decides ? s_alpha
                                        : __ldcg(&alpha[bb * c.Hkv + hs]);
        const bool evict = shifted_mark(c, li, t, !c.disable && a > 0.0f);
        c.slot_pos[li * c.cap + slot] = t;
        c.ring[li * c.w + t % c.w] = slot | (evict ? static_cast<int>(RING_EVICT) : 0);
        if (!(flags & 1)) c.count[li] = cnt_new;
      }
    } else if (lane == 0) {
      set_status(c.ctrl, (flags & 4) ? DMS_ST_CAPACITY : DMS_ST_POOL_EXHAUSTED);
    }
    int last = 0;
    if (lane == 0) {
      // plan of the next append (token t + 1), from the values just written
      *plan_at(c, li, t + 1) = make_plan(s_ring_next, t + 1, cnt_new, np_new, c);
      // the owners count the step (every CTA of the cluster has read the page
      // counter and the positions before its partial landed here)
      last = count_step(c, ok && (flags & 2) ? 1 : 0, static_cast<int>(gridDim.x) / cs, next_page0) ? 1 : 0;
    }
    if (__shfl_sync(0xffffffffu, last, 0)) advance_positions(c, layer, lane, 32, nl);
    return;
  }

  // the head's output rows: per row the weights of the cs partials (each
  // thread for its own row, from the partials' maxima and sums), then O / L,
  // four consecutive elements of one row per thread and pass; the merging
  // threads are warps 0-2 in a fused step (warp 3 counts the step), else all
  if (landed) {
    constexpr int kMergeThreads = FUSED ? kThreads - 32 : kThreads;
    __nv_bfloat16* ob = o + (static_cast<long>(bb) * c.Hq + static_cast<long>(h) * g) * D;
    const bool vec_out = (reinterpret_cast<uintptr_t>(ob) & 7) == 0;
    for (int e4 = tid; e4 < g * (D / 4); e4 += kMergeThreads) {
      const int r = e4 / (D / 4), d = 4 * (e4 % (D / 4));
      float mk[kPickCluster], M = -INFINITY;
#pragma unroll
      for (int k = 0; k < kPickCluster; ++k) {
        mk[k] = k < cs ? inbox[(k * g + r) * IMLD + D] : -INFINITY;
        M = fmaxf(M, mk[k]);
      }
      const float Mu = M == -INFINITY ? 0.f : M;
      float L = 0.f;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < kPickCluster; ++k) {
        if (k < cs) {
          const float wgt = ex2_fast(mk[k] - Mu);
          L = fmaf(wgt, inbox[(k * g + r) * IMLD + D + 1], L);
          const float4 v = *reinterpret_cast<const float4*>(inbox + (k * g + r) * IMLD + d);
          a.x = fmaf(wgt, v.x, a.x);
          a.y = fmaf(wgt, v.y, a.y);
          a.z = fmaf(wgt, v.z, a.z);
          a.w = fmaf(wgt, v.w, a.w);
        }
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const uint32_t lo = pack_bf16(a.x * inv, a.y * inv), hi = pack_bf16(a.z * inv, a.w * inv);
      if (vec_out) {
        *reinterpret_cast<uint2*>(ob + r * D + d) = make_uint2(lo, hi);
      } else {
        const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(&lo);
        const __nv_bfloat16* ph = reinterpret_cast<const __nv_bfloat16*>(&hi);
        ob[r * D + d] = pb[0];
        ob[r * D + d + 1] = pb[1];
        ob[r * D + d + 2] = ph[0];
        ob[r * D + d + 3] = ph[1];
      }
    }
  }
}

// Largest cluster (a power of two <= 8) the device co-schedules at `mper`
// stages per warp, and the CTAs per SM (1 or 2) its shared memory allows.
template <int D, bool FP8, bool FUSED, bool TQ>
static void cluster_limits(int g, int mper, int* max_cs, int* per_sm) {
  *max_cs = 1;
  *per_sm = 1;
  int dev = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  for (int cs = kPickCluster; cs > 1; cs >>= 1) {
    const size_t smem = ClusterSmem<D, FP8, TQ>::bytes(g, cs, mper);
    if (smem + 4096 > static_cast<size_t>(optin)) continue;  // static shared memory on top
    if (cudaFuncSetAttribute(k_decode_cluster<D, FP8, FUSED, TQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess) {
      cudaGetLastError();
      continue;
    }
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
    if (cudaOccupancyMaxActiveClusters(&n, k_decode_cluster<D, FP8, FUSED, TQ>, &cfg) == cudaSuccess && n > 0) {
      *max_cs = cs;
      int nb = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_decode_cluster<D, FP8, FUSED, TQ>, kThreads, smem) ==
              cudaSuccess &&
          nb > 1)
        *per_sm = 2;
      cudaGetLastError();
      return;
    }
    cudaGetLastError();
  }
}

// Cluster size and stages per warp: the largest power of two cs with
// cs * heads <= k * SMs (k the CTAs per SM the shared memory allows), at the
// full stage count, or at half of it when that fits more CTAs per SM and so
// gives a larger cluster, or when there are more heads than SMs (one CTA per
// head; more CTAs share each SM).
template <int D, bool FP8, bool FUSED, bool TQ>
static void pick_cluster(int heads, int g, int num_sms, int* cs_out, int* mper_out) {
  using S = ClusterSmem<D, FP8, TQ>;
  static int lim[17][4] = {{0}};  // by g (<= 16): max cs and CTAs per SM at MPER, then at MPER / 2
  int* l = lim[g < 16 ? g : 16];
  if (l[0] == 0) {
    cluster_limits<D, FP8, FUSED, TQ>(g, S::MPER, &l[0], &l[1]);
    cluster_limits<D, FP8, FUSED, TQ>(g, (S::MPER + 1) / 2, &l[2], &l[3]);
  }
  auto size = [&](int m, int k) {
    int cs = 1;
    while (cs * 2 <= m && static_cast<long>(cs) * 2 * heads <= static_cast<long>(k) * num_sms) cs *= 2;
    return cs;
  };
  const int full = size(l[0], l[1]), half = size(l[2], l[3]);
  if (half > full || heads > num_sms) {
    *cs_out = half;
    *mper_out = (S::MPER + 1) / 2;
  } else {
    *cs_out = full;
    *mper_out = S::MPER;
  }
}

template <int D, bool FP8, bool FUSED, bool TQ>
static cudaError_t launch_cluster_t(const CacheView& c, int layer, const void* q, void* o, const void* k,
                                   const void* v, float* alpha, const DecideArgs* da, const CUtensorMap* kmap,
                                   const CUtensorMap* vmap, int num_sms, cudaStream_t s, bool early, int nl) {
  const int g = c.Hq / c.Hkv;
  auto kern = k_decode_cluster<D, FP8, FUSED, TQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  const int heads = nl * c.B * c.Hkv;
  int cs = 1, mper = 1;
  pick_cluster<D, FP8, FUSED, TQ>(heads, g, num_sms, &cs, &mper);
  const size_t smem = ClusterSmem<D, FP8, TQ>::bytes(g, cs, mper);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(cs * heads, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  DecideArgs none{};
  return cudaLaunchKernelEx(&cfg, kern, c, layer, nl, early ? 1 : 0, static_cast<const __nv_bfloat16*>(q),
                            static_cast<__nv_bfloat16*>(o), cs, mper, static_cast<const __nv_bfloat16*>(k),
                            static_cast<const __nv_bfloat16*>(v), alpha, da ? *da : none, da ? 1 : 0, *kmap, *vmap);
}

// One instantiation per (head dim, page type, fused step, key-major tiles).
template <bool FP8, bool FUSED>
static cudaError_t launch_cluster_dt(const CacheView& c, int layer, const void* q, void* o, const void* k,
                                    const void* v, float* alpha, const DecideArgs* da, const CUtensorMap* kmap,
                                    const CUtensorMap* vmap, int num_sms, cudaStream_t s, bool early, int nl) {
  const bool tq = c.Hq / c.Hkv <= 8;
  if (c.D == 64)
    return tq ? launch_cluster_t<64, FP8, FUSED, true>(c, layer, q, o, k, v, alpha, da, kmap, vmap, num_sms, s, early,
                                                       nl)
              : launch_cluster_t<64, FP8, FUSED, false>(c, layer, q, o, k, v, alpha, da, kmap, vmap, num_sms, s,
                                                        early, nl);
  return tq ? launch_cluster_t<128, FP8, FUSED, true>(c, layer, q, o, k, v, alpha, da, kmap, vmap, num_sms, s, early,
                                                      nl)
            : launch_cluster_t<128, FP8, FUSED, false>(c, layer, q, o, k, v, alpha, da, kmap, vmap, num_sms, s, early,
                                                       nl);
}

int decode_cluster_box_rows(int D, bool fp8) { return cluster_rows(D, fp8); }

cudaError_t launch_decode_cluster(const CacheView& c, int layer, const void* q, void* o, bool fused, const void* k,
                                  const void* v, float* alpha, const DecideArgs* fused_decide, const CUtensorMap* kmap,
                                  const CUtensorMap* vmap, int num_sms, cudaStream_t s, bool early, int nl) {
  if (!kmap || !vmap || c.kv_dtype == DMS_F32 || nl < 1) return cudaErrorInvalidValue;
  if (fused)
    return c.kv_dtype == DMS_FP8_E4M3
               ? launch_cluster_dt<true, true>(c, layer, q, o, k, v, alpha, fused_decide, kmap, vmap, num_sms, s, early,
                                               nl)
               : launch_cluster_dt<false, true>(c, layer, q, o, k, v, alpha, fused_decide, kmap, vmap, num_sms, s,
                                                early, nl);
  if (c.kv_dtype == DMS_FP8_E4M3)
    return launch_cluster_dt<true, false>(c, layer, q, o, k, v, alpha, nullptr, kmap, vmap, num_sms, s, early, nl);
  return launch_cluster_dt<false, false>(c, layer, q, o, k, v, alpha, nullptr, kmap, vmap, num_sms, s, early, nl);
}

}  // namespace dms

