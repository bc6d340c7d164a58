// DMS-masked prefill attention on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory).
//
// Visible set of query i ([DMS-Qwen3], attention: the training score_mod's
// window and eviction gate at their hard inference limit):
//   V_i = { j <= i : i - j < w  or  alpha_j <= 0 }
// = band (i - w < j <= i)  U  kept prefix (j <= i - w, alpha_j <= 0).
//
// A CTA owns two Q tiles of 128 rows; a Q tile is NP = 128/g consecutive
// positions x the g query heads that share one KV head (row t = p * g + r),
// so every K/V tile feeds 2 x 128 rows.  Key tiles of 64 come from the
// contiguous band [i0 - w + 1, i1 - 1] of the CTA's 2 NP positions and from
// the position-sorted kept list; evicted keys outside the window are never
// loaded.  Warp roles:
//   K loader   : TMA (no multicast) of the Q tiles, then K of every key tile
//                into a ring of stages (band tiles straight from the input
//                rows, kept tiles from the kept copy written by the
//                compaction); a K stage is free again once both Q tiles'
//                scores are computed;
//   V loader   : V of every key tile into its own ring, free again once both
//                Q tiles' P V are done;
//   MMA warps  : one per Q tile w: S_w = Q_w K^T (tcgen05.mma M=128, N=64,
//                K=16 x D/16, both K-major in 128-byte-swizzled shared memory,
//                S_w in TMEM) and O_w += P_w V (P_w in TMEM as bf16, V
//                MN-major in shared memory, O_w in TMEM), in the order
//                S_w(t+1), PV_w(t): each Q tile's next scores run on the tensor
//                cores while its softmax of tile t runs, and the two Q tiles
//                proceed independently;
//   softmax    : one warpgroup per Q tile, one thread per row; a row's
//                visible keys in a tile are one column range (the band is
//                contiguous in position; the kept list is position-sorted, so
//                the keys at or before i - w are its first kept_upto(i-w+1)
//                entries), applied as a bit mask; the exponent
//                reference of a row is raised only when a tile's max exceeds
//                it by 2^8, so O is rescaled rarely (O / l is exact either
//                way).
// mbarriers order every hand-off (loads, S ready / S read, P ready, P V done,
// stage free); every wait is bounded.
#include "dms_internal.cuh"

namespace dms {


constexpr int kPfRows = 128;     // query rows per Q tile (TMEM lanes)
constexpr int kPfQT = 2;         // Q tiles per CTA
constexpr int kPfBN = 64;        // keys per K/V tile
constexpr int kPfMmaWarp = 8;    // warps 0-3: softmax of Q tile 0, 4-7: Q tile 1; 8, 9: MMA issue for
                                 // Q tile 0, 1
constexpr int kPfLoadWarp = 10;  // 10: Q and K loads, 11: V loads
constexpr int kPfThreads = 384;

template <int D>
struct PfSmem {
  static constexpr int HALVES = D / 64;
  static constexpr int Q_BYTES = HALVES * kPfRows * 128;  // one Q tile: [half][128 rows][128 B]
  static constexpr int KV_BYTES = HALVES * kPfBN * 128;   // K (or V) of one key tile: [half][64 keys][128 B]
  static constexpr int ST = D == 64 ? 8 : 3;              // K stages, V stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + kPfQT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + ST * KV_BYTES;
  static constexpr int O_BYTES = HALVES * kPfRows * 128;  // per Q tile: O / l (bf16), staged for the TMA stores
  static constexpr int OFF_O = OFF_V + ST * KV_BYTES;
  static constexpr int BYTES = OFF_O + kPfQT * O_BYTES;
  // tensor memory: S0, S1 (64 fp32 columns each), O0, O1 (D columns each),
  // P0, P1 (64 bf16 = 32 columns each)
  static constexpr uint32_t COL_O = 2 * kPfBN;
  static constexpr uint32_t COL_P = COL_O + 2 * D;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(COL_P + kPfQT * kPfBN / 2 <= TMEM_COLS, "tensor memory columns");
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Named barriers among the two softmax warpgroups (ids 1, 2; 0 is
// __syncthreads): arrive without waiting, or wait for `count` arrivals.
template <int ID>
__device__ __forceinline__ void named_arrive() {
  asm volatile("bar.arrive %0, %1;\n" ::"n"(ID), "n"(2 * kPfRows) : "memory");
}
template <int ID>
__device__ __forceinline__ void named_sync() {
  asm volatile("bar.sync %0, %1;\n" ::"n"(ID), "n"(2 * kPfRows) : "memory");
}

// the 128 threads of softmax warpgroup qt (ids 3, 4)
__device__ __forceinline__ void wg_sync(int qt) {
  if (qt == 0)
    asm volatile("bar.sync 3, %0;\n" ::"n"(kPfRows) : "memory");
  else
    asm volatile("bar.sync 4, %0;\n" ::"n"(kPfRows) : "memory");
}

// 4-D TMA tile store from shared memory (bulk group), its commit and waits
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* smem_src, int c0, int c1, int c2,
                                             int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];\n" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(smem_src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));  // stays between the turn barriers
  return y;
}

// paired fp32 arithmetic (one instruction for two lanes of a 64-bit pair)
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 32 consecutive fp32 columns of this thread's TMEM lane, without waiting.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// 3-D TMA tile load (no multicast).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];\n" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// One work item: a block of kPfQT * NP query rows of one (batch, KV head);
// i0, i1 index the call's rows, whose positions are T0 + i.  Its key tiles:
// nkt kept-list tiles, npre band tiles of positions [jlo, T0) from the window
// copy (a later chunk of a chunked prefill only), then the band tiles of the
// call's own positions [jin, jhi].
struct PfItem {
  int h, b, bh, i0, i1, nk, jlo, jhi, jin, nkt, npre, ntiles;
  bool valid;
};

// The k-th item of CTA `cta` of G: items are numbered heaviest (latest
// block) first and dealt in snake order, one per CTA per round, so the
// rounds' decreasing weights even out across CTAs.
__device__ __forceinline__ int pf_item_index(int k, int G, int cta) {
  return k * G + ((k & 1) ? (G - 1 - cta) : cta);
}

// The item's geometry; nk (kept keys before i1 - w, a table read) is passed in
// so that callers can fetch it one item ahead.
__device__ __forceinline__ PfItem pf_item(const CacheView& c, int T0, int T, int NP, int nblk, int nitems, int u,
                                          int nk) {
  PfItem it{};
  it.valid = u < nitems;
  if (!it.valid) return it;
  const int per = c.Hkv * c.B, blk = nblk - 1 - u / per, rem = u % per;
  it.h = rem % c.Hkv;
  it.b = rem / c.Hkv;
  it.bh = it.b * c.Hkv + it.h;
  it.i0 = blk * kPfQT * NP;
  it.i1 = min(T, it.i0 + kPfQT * NP);
  it.nk = nk;
  it.jlo = max(0, T0 + it.i0 - c.w + 1);  // band positions [jlo, jhi]
  it.jhi = T0 + it.i1 - 1;
  it.jin = max(it.jlo, T0);
  it.nkt = (it.nk + kPfBN - 1) / kPfBN;  // kept tiles
  it.npre = it.jlo < T0 ? (min(T0, it.jhi + 1) - it.jlo + kPfBN - 1) / kPfBN : 0;
  it.ntiles = it.nkt + it.npre + (it.jhi - it.jin + kPfBN) / kPfBN;
  return it;
}

// Position of the first key of tile j of an item, and its source (0: kept
// copy, 1: window copy, 2: the call's own rows).
__device__ __forceinline__ int pf_tile(const PfItem& it, int j, int& src) {
  if (j < it.nkt) {
    src = 0;
    return j * kPfBN;  // a kept-list rank
  }
  if (j < it.nkt + it.npre) {
    src = 1;
    return it.jlo + (j - it.nkt) * kPfBN;
  }
  src = 2;
  return it.jin + (j - it.nkt - it.npre) * kPfBN;
}

// A table read issued where it is written (the asm keeps the compiler from
// sinking it to its use, an item later), and the point from which its value
// may be used (keeps the compiler from consuming it early, which would make
// the warp wait for the read right after issuing it).
__device__ __forceinline__ int ld_early_i32(const int* p) {
  int v;
  asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ int use_late(int v) {
  int r;
  asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}

// kept_upto(bh, x) of item u's (batch, KV head) at position x = T0 + i0 + dx
// (0 when x <= 0 or the item does not exist; x is clamped to T0 + T).  In the
// soft (training) mode every key is a prefix key: kept_upto(x) = x.
__device__ __forceinline__ int pf_kept_upto(const CacheView& c, int T0, int T, int NP, int nblk, int nitems, int u,
                                           int dx, bool soft) {
  if (u >= nitems) return 0;
  const int per = c.Hkv * c.B, blk = nblk - 1 - u / per, rem = u % per;
  const int x = min(T0 + blk * kPfQT * NP + dx, T0 + T);
  if (soft) return max(x, 0);
  return x > 0 ? ld_early_i32(c.kept_upto + static_cast<long>((rem / c.Hkv) * c.Hkv + rem % c.Hkv) * (c.max_pos + 1) + x)
               : 0;
}

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
    k_attn_prefill_tc(CacheView c, int T0, int T, __nv_bfloat16* o, const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ CUtensorMap kkmap, const __grid_constant__ CUtensorMap kvmap,
                      const __grid_constant__ CUtensorMap wkmap, const __grid_constant__ CUtensorMap wvmap,
                      const __grid_constant__ CUtensorMap omap, const float* pen,
                      const __grid_constant__ CUtensorMap penmap, int pen_tma) {
  using L = PfSmem<D>;
  constexpr int ST = L::ST;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sb = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint32_t tmem_base;
  __shared__ __align__(8) uint64_t bar_q, q_empty, k_full[ST], v_full[ST], k_empty[ST], v_empty[ST];
  __shared__ __align__(8) uint64_t s_full[kPfQT], s_free[kPfQT], p_full[kPfQT], pv_done[kPfQT], o_free[kPfQT];
  __shared__ int s_abort;
  // anchors of the exponentials' turn: a zero read after the turn begins and
  // every row's sum written (to one word per group) before it ends (a barrier
  // orders memory accesses only, so the exponentials are tied to it through
  // these)
  __shared__ float s_turn_zero;
  __shared__ float s_turn_sink[kPfQT];
  // soft mode: the penalties of each V stage's prefix keys, loaded with the
  // V tile (the stage is free again only after P V, so after the softmax used them)
  __shared__ __align__(128) float s_pen[ST][kPfBN];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = c.Hq / c.Hkv, NP = kPfRows / g, w = c.w;
  // soft mode (training attention, pen != null): every key at or before i - w
  // is a prefix key read from the input rows, its score raised by pen[key]
  const bool soft = pen != nullptr;
  const int nblk = (T + kPfQT * NP - 1) / (kPfQT * NP);
  const int nitems = nblk * c.Hkv * c.B, G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
  // item k of this CTA, and its nk (kept keys before i1 - w)
  auto item_nk = [&](int k) {
    const int u = pf_item_index(k, G, cta);
    if (u >= nitems) return 0;
    const int i0 = (nblk - 1 - u / (c.Hkv * c.B)) * kPfQT * NP, i1 = min(T, i0 + kPfQT * NP);
    return pf_kept_upto(c, T0, T, NP, nblk, nitems, u, i1 - i0 - w, soft);
  };
  auto item = [&](int k, int nk) { return pf_item(c, T0, T, NP, nblk, nitems, pf_item_index(k, G, cta), nk); };

  if (tid == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&q_empty, kPfQT);  // both Q tiles' last scores of the item done
    for (int i = 0; i < ST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], kPfQT);  // both Q tiles' scores done with the K stage
      mbar_init(&v_empty[i], kPfQT);  // both Q tiles' P V done with the V stage
    }
    for (int i = 0; i < kPfQT; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);  // one arrival per softmax warp
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&o_free[i], 4);  // O of the item read out: the next item may start a fresh sum
    }
    fence_mbar_init();
    s_abort = 0;
    s_turn_zero = 0.f;
  }
  if (warp == kPfMmaWarp) tmem_alloc(&tmem_base, L::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  auto give_up = [&]() {
    set_status(c.ctrl, DMS_ST_TIMEOUT);
    s_abort = 1;
  };

  if (warp == kPfLoadWarp) {
    // ---- per item: Q (once the previous item's scores are done), then K of
    // every key tile -----------------------------------------------------------
    if (lane == 0) {
      int t = 0;  // tiles loaded so far (ring position)
      PfItem it = item(0, item_nk(0));
      for (int k = 0; it.valid && !s_abort; ++k) {
        const int nk_next = item_nk(k + 1);
        if (k > 0 && !mbar_wait_parked(&q_empty, (k - 1) & 1)) {
          give_up();
          break;
        }
        mbar_expect_tx(&bar_q, kPfQT * L::Q_BYTES);
        for (int qt = 0; qt < kPfQT; ++qt)
          for (int hf = 0; hf < L::HALVES; ++hf)
            tma_load_3d(sb + L::OFF_Q + qt * L::Q_BYTES + hf * (kPfRows * 128), &qmap, hf * 64, it.h * g,
                        it.b * T + it.i0 + qt * NP, &bar_q);
        for (int j = 0; j < it.ntiles; ++j, ++t) {
          const int st = t % ST, use = t / ST;
          if (use > 0 && !mbar_wait_parked(&k_empty[st], (use - 1) & 1)) {
            give_up();
            break;
          }
          int src;
          const int jb = pf_tile(it, j, src);
          mbar_expect_tx(&k_full[st], L::KV_BYTES);
          for (int hf = 0; hf < L::HALVES; ++hf) {
            unsigned char* dk = sb + L::OFF_K + st * L::KV_BYTES + hf * (kPfBN * 128);
            if (src == 0 && soft)
              tma_load_3d(dk, &kmap, hf * 64, it.h, it.b * T + jb, &k_full[st]);
            else if (src == 0)
              tma_load_2d(dk, &kkmap, hf * 64, it.bh * c.max_pos + jb, &k_full[st]);
            else if (src == 1)
              tma_load_2d(dk, &wkmap, hf * 64, it.bh * w + (jb - (T0 - w)), &k_full[st]);
            else
              tma_load_3d(dk, &kmap, hf * 64, it.h, it.b * T + (jb - T0), &k_full[st]);
          }
        }
        it = item(k + 1, use_late(nk_next));
      }
    }
  } else if (warp == kPfLoadWarp + 1) {
    // ---- V of every key tile of every item ------------------------------
    if (lane == 0) {
      int t = 0;
      PfItem it = item(0, item_nk(0));
      for (int k = 0; it.valid && !s_abort; ++k) {
        const int nk_next = item_nk(k + 1);
        for (int j = 0; j < it.ntiles; ++j, ++t) {
          const int st = t % ST, use = t / ST;
          if (use > 0 && !mbar_wait_parked(&v_empty[st], (use - 1) & 1)) {
            give_up();
            break;
          }
          int src;
          const int jb = pf_tile(it, j, src);
          const bool pen_tile = soft && pen_tma && src == 0;
          mbar_expect_tx(&v_full[st], L::KV_BYTES + (pen_tile ? kPfBN * 4 : 0));
          if (pen_tile) tma_load_2d(&s_pen[st][0], &penmap, jb, it.bh, &v_full[st]);
          for (int hf = 0; hf < L::HALVES; ++hf) {
            unsigned char* dv = sb + L::OFF_V + st * L::KV_BYTES + hf * (kPfBN * 128);
            if (src == 0 && soft)
              tma_load_3d(dv, &vmap, hf * 64, it.h, it.b * T + jb, &v_full[st]);
            else if (src == 0)
              tma_load_2d(dv, &kvmap, hf * 64, it.bh * c.max_pos + jb, &v_full[st]);
            else if (src == 1)
              tma_load_2d(dv, &wvmap, hf * 64, it.bh * w + (jb - (T0 - w)), &v_full[st]);
            else
              tma_load_3d(dv, &vmap, hf * 64, it.h, it.b * T + (jb - T0), &v_full[st]);
          }
        }
        it = item(k + 1, use_late(nk_next));
      }
    }
  } else if (warp == kPfMmaWarp || warp == kPfMmaWarp + 1) {
    // ---- tensor-core issue for Q tile qt (one thread) ----------------------
    const int qt = warp - kPfMmaWarp;
    if (lane == 0) {
      constexpr uint32_t IDESC_S = umma_idesc_bf16(kPfRows, kPfBN, 0);
      constexpr uint32_t IDESC_O = umma_idesc_bf16(kPfRows, D, 1);
      // S(t) = Q K(t)^T; after the item's last scores Q may be replaced
      auto issue_s = [&](int t, bool last_of_item) -> bool {
        const int st = t % ST;
        if (!mbar_wait_bounded(&k_full[st], (t / ST) & 1)) return false;
        tc_fence_after();
        const uint32_t qa = smem_u32(sb + L::OFF_Q + qt * L::Q_BYTES);
        const uint32_t ka = smem_u32(sb + L::OFF_K + st * L::KV_BYTES);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t qoff = (ks / 4) * (kPfRows * 128) + (ks % 4) * 32;
          const uint32_t koff = (ks / 4) * (kPfBN * 128) + (ks % 4) * 32;
          umma_bf16(tmem + qt * kPfBN, umma_desc_sw128(qa + qoff, 16, 1024), umma_desc_sw128(ka + koff, 16, 1024),
                    IDESC_S, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[qt]);
        umma_commit(&k_empty[st]);  // this Q tile is done with the K stage
        if (last_of_item) umma_commit(&q_empty);
        return true;
      };
      // O += P(t) V(t); the item's first product starts a fresh sum once the
      // previous item's O has been read out
      auto issue_pv = [&](int t, int j, int k) -> bool {
        const int st = t % ST;
        if (!mbar_wait_bounded(&v_full[st], (t / ST) & 1)) return false;
        if (!mbar_wait_bounded(&p_full[qt], t & 1)) return false;
        if (j == 0 && k > 0 && !mbar_wait_bounded(&o_free[qt], (k - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t va = smem_u32(sb + L::OFF_V + st * L::KV_BYTES);
#pragma unroll
        for (int ks = 0; ks < kPfBN / 16; ++ks)
          umma_bf16_ts(tmem + L::COL_O + qt * D, tmem + L::COL_P + qt * (kPfBN / 2) + ks * 8,
                       umma_desc_sw128(va + ks * 16 * 128, kPfBN * 128, 1024), IDESC_O, (j > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&pv_done[qt]);
        umma_commit(&v_empty[st]);  // this Q tile is done with the V stage
        return true;
      };
      int t = 0;
      PfItem it = item(0, item_nk(0));
      bool ok = !it.valid || (mbar_wait_bounded(&bar_q, 0) && issue_s(0, it.ntiles == 1));
      for (int k = 0; ok && it.valid; ++k) {
        const PfItem nx = item(k + 1, item_nk(k + 1));  // (used at the item's last tile)
        for (int j = 0; ok && j < it.ntiles; ++j, ++t) {
          // within the item: the next scores once the softmax has read S(t),
          // then P(t) V(t); at its last tile P V first (the epilogue waits for
          // it), then the next item's first scores
          if (j + 1 < it.ntiles) {
            ok = mbar_wait_bounded(&s_free[qt], t & 1) && issue_s(t + 1, j + 2 == it.ntiles);
            ok = ok && issue_pv(t, j, k);
          } else {
            ok = issue_pv(t, j, k);
            if (nx.valid)
              ok = ok && mbar_wait_bounded(&s_free[qt], t & 1) && mbar_wait_bounded(&bar_q, (k + 1) & 1) &&
                   issue_s(t + 1, nx.ntiles == 1);
          }
          if (s_abort) ok = false;
        }
        it = nx;
      }
      if (!ok) give_up();
    }
  } else {
    // ---- softmax: warpgroup qt, one thread per row ---------------------------
    const int qt = warp >> 2, row = tid & (kPfRows - 1);
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tmem_s = tmem + lane_off + qt * kPfBN;
    const uint32_t tmem_o = tmem + lane_off + L::COL_O + qt * D;
    const uint32_t tmem_p = tmem + lane_off + L::COL_P + qt * (kPfBN / 2);
    const int p_row = qt * NP + row / g;  // the row's position within the item
    const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    // the row's count of visible kept keys: kept-list entries [0, ck) are the
    // positions <= i - w
    auto kept_visible = [&](int k) {
      return pf_kept_upto(c, T0, T, NP, nblk, nitems, pf_item_index(k, G, cta), p_row - w + 1, soft);
    };
    bool ok = true;
    int t = 0;
    PfItem it = item(0, item_nk(0));
    int ck = kept_visible(0);
    // The two warpgroups take turns for the exponentials (named barrier 1:
    // WG1 may start, 2: WG0 may start; bar.arrive by the group that finishes,
    // bar.sync by the one that waits), so one group's exponentials overlap the
    // other group's tensor-core work and bookkeeping.  Both groups walk the
    // same items and tiles, and every barrier step runs even after a failed
    // wait, so neither group can be left waiting.
    for (int k = 0; it.valid; ++k) {
      const int nk_next = item_nk(k + 1), ck_next = kept_visible(k + 1);
      const int i_row = T0 + it.i0 + p_row;                               // the row's position
      const int blo = max(0, i_row - w + 1), bhi = min(i_row, it.jhi);  // band positions of the row
      float m_ref = -INFINITY, l_row = 0.f;
      for (int j = 0; j < it.ntiles; ++j, ++t) {
        // visible columns [c_lo, c_hi] of this tile for the row
        int src;
        const int jb = pf_tile(it, j, src);
        const bool kt = src == 0;
        // window-copy tiles end before the call's first position T0
        const int hi = src == 1 ? min(bhi, T0 - 1) : bhi;
        const int c_lo = max(kt ? 0 : blo - jb, 0), c_hi = min(kt ? ck - 1 - jb : hi - jb, kPfBN - 1);
        const bool row_full = c_lo == 0 && c_hi == kPfBN - 1;
        ok = ok && mbar_wait_bounded(&s_full[qt], t & 1);
        tc_fence_after();
        uint32_t sr[kPfBN];
        if (ok) {
          tmem_ld32_nowait(tmem_s, sr);
          tmem_ld32_nowait(tmem_s + 32, sr + 32);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int n = 0; n < kPfBN; ++n) sr[n] = 0u;
        }
        tc_fence_before();
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(&s_free[qt]);  // S may be overwritten by the next tile's scores
        // raw scores with the invisible ones at -inf; row max over 4 chains
        float sv[kPfBN];
        if (__all_sync(0xffffffffu, row_full)) {
#pragma unroll
          for (int n = 0; n < kPfBN; ++n) sv[n] = __uint_as_float(sr[n]);
        } else {
          // bits c_lo..c_hi (none when the range is empty)
          uint32_t m0 = 0u, m1 = 0u;
          if (c_lo <= c_hi) {
            const unsigned long long m = (~0ull >> (kPfBN - 1 - (c_hi - c_lo))) << c_lo;
            m0 = static_cast<uint32_t>(m);
            m1 = static_cast<uint32_t>(m >> 32);
          }
#pragma unroll
          for (int n = 0; n < kPfBN; ++n)
            sv[n] = (((n < 32 ? m0 : m1) >> (n & 31)) & 1u) ? __uint_as_float(sr[n]) : -INFINITY;
        }
        if (soft && kt && c_lo <= c_hi) {
          // penalty of the prefix keys, in raw-score units (the softmax works
          // in s * log2(e) / sqrt(D)): from the V stage, else from global memory
          const float rs = sqrtf(static_cast<float>(D));
          if (pen_tma) {
            const int st = t % ST;
            ok = ok && mbar_wait_bounded(&v_full[st], (t / ST) & 1);
            // (16-byte loads of the row every lane reads alike)
            const float4* pr = reinterpret_cast<const float4*>(&s_pen[st][0]);
#pragma unroll
            for (int n4 = 0; n4 < kPfBN / 4; ++n4) {
              const float4 pv = pr[n4];
              const float pe[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int n = 4 * n4 + e;
                if (n >= c_lo && n <= c_hi) sv[n] = fmaf(pe[e], rs, sv[n]);
              }
            }
          } else {
            const float* pr = pen + static_cast<long>(it.bh) * T + jb;
#pragma unroll
            for (int n = 0; n < kPfBN; ++n)
              if (n >= c_lo && n <= c_hi) sv[n] = fmaf(__ldg(pr + n), rs, sv[n]);
          }
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < kPfBN; n += 2) mx4[(n >> 1) & 3] = fmax3(mx4[(n >> 1) & 3], sv[n], sv[n + 1]);
        const float tmax = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
        // raise the reference only when this tile exceeds it by more than 2^8
        const bool raise = tmax > m_ref + 8.0f;
        float factor = 1.0f;
        if (raise) {
          factor = (m_ref == -INFINITY) ? 0.0f : ex2_approx(m_ref - tmax);
          m_ref = tmax;
          l_row *= factor;
        }
        const float m_use = m_ref == -INFINITY ? 0.f : m_ref;  // a fully masked row so far: all p = 0
        if (qt == 0) {
          if (t > 0) named_sync<2>();
        } else {
          named_sync<1>();
        }
        const float neg_m = *reinterpret_cast<volatile float*>(&s_turn_zero) - m_use;
        const uint64_t nm2 = f2_pack(neg_m, neg_m);
        uint32_t pk[kPfBN / 2];
        uint64_t ps4[4] = {0ull, 0ull, 0ull, 0ull};  // pairs of +0.0f
#pragma unroll
        for (int e = 0; e < kPfBN / 2; ++e) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(sv[2 * e], sv[2 * e + 1]), sl2x2, nm2), x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          ps4[e & 3] = f2_add(ps4[e & 3], f2_pack(p0, p1));
          pk[e] = pack_bf16(p0, p1);
        }
        float s_even, s_odd;
        f2_unpack(f2_add(f2_add(ps4[0], ps4[1]), f2_add(ps4[2], ps4[3])), s_even, s_odd);
        const float psum = s_even + s_odd;
        *reinterpret_cast<volatile float*>(&s_turn_sink[qt]) = psum;
        // the turn ends once every exponential is done: the arrive is control
        // dependent on their sum (the condition always holds: psum is a sum of
        // non-negative terms, never this negative NaN pattern)
        if (__float_as_uint(psum) != 0xFFFFFFFFu) {
          if (qt == 0)
            named_arrive<1>();
          else
            named_arrive<2>();
        }
        l_row += psum;
        // P V of the previous tile has finished with P and with O (for the
        // item's first tile the previous item's epilogue waited for it)
        if (j > 0) ok = ok && mbar_wait_bounded(&pv_done[qt], (t - 1) & 1);
        tc_fence_after();
        if (ok && j > 0 && __any_sync(0xffffffffu, raise && factor != 1.0f)) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            float ov[32];
            tmem_ld32(tmem_o + c0, ov);
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) ov[jj] *= factor;
            tmem_st32(tmem_o + c0, ov);
          }
        }
        tmem_st32_nowait(tmem_p, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();  // the warp's P rows and O rescale precede lane 0's release
        if (ok && lane == 0) mbar_arrive(&p_full[qt]);
        if (s_abort) ok = false;
      }
      // the item's last P V, then O / l; O is released to the next item as
      // soon as it is in registers
      ok = ok && mbar_wait_bounded(&pv_done[qt], (t - 1) & 1);
      tc_fence_after();
      // read O, release it, write O / l (bf16, 64-column boxes) to this
      // group's staging tile once the previous item's TMA stores have read
      // it, and store it with the TMA (rows at or past T are clipped by the
      // map)
      const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
      unsigned char* stg = sb + L::OFF_O + qt * L::O_BYTES;
      const bool store = ok && it.i0 + qt * NP < T;
      if (store) {
        if (row == 0) bulk_wait_read0();  // the previous item's stores have read the staging tile
        wg_sync(qt);
      }
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float ov[32];
        if (ok) tmem_ld32(tmem_o + c0, ov);
        if (store) {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int e = ch * 8;
            *reinterpret_cast<uint4*>(stg + (c0 / 64) * (kPfRows * 128) + swz(row, (c0 % 64) / 8 + ch)) =
                make_uint4(pack_bf16(ov[e] * inv, ov[e + 1] * inv), pack_bf16(ov[e + 2] * inv, ov[e + 3] * inv),
                           pack_bf16(ov[e + 4] * inv, ov[e + 5] * inv), pack_bf16(ov[e + 6] * inv, ov[e + 7] * inv));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&o_free[qt]);
      if (store) {
        fence_proxy_async();  // the tile visible to the TMA
        wg_sync(qt);
        if (row == 0) {
          for (int hf = 0; hf < L::HALVES; ++hf)
            tma_store_4d(&omap, stg + hf * (kPfRows * 128), hf * 64, it.h * g, it.i0 + qt * NP, it.b);
          bulk_commit();
        }
      }
      it = item(k + 1, use_late(nk_next));
      ck = use_late(ck_next);
    }
    if (qt == 0 && t > 0) named_sync<2>();  // WG1's last hand-back
    if (row == 0) bulk_wait0();                 // this group's stores complete before the CTA ends
    if (!ok && row == 0) give_up();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kPfMmaWarp) tmem_dealloc(tmem, L::TMEM_COLS);
}

template <int D>
static cudaError_t launch_tc(const CacheView& c, int T0, int T, void* o, const PrefillMaps& m, cudaStream_t s,
                             const float* pen, const CUtensorMap* penmap) {
  const size_t smem = PfSmem<D>::BYTES + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_attn_prefill_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int g = c.Hq / c.Hkv, NP = kPfRows / g;
  const long nitems = static_cast<long>((T + kPfQT * NP - 1) / (kPfQT * NP)) * c.Hkv * c.B;
  const int grid = static_cast<int>(min(nitems, static_cast<long>(c.num_sms)));  // persistent: one CTA per SM
  k_attn_prefill_tc<D><<<grid, kPfThreads, smem, s>>>(c, T0, T, static_cast<__nv_bfloat16*>(o), m.q, m.k, m.v,
                                                      m.kept_k, m.kept_v, m.win_k, m.win_v, m.o, pen,
                                                      penmap ? *penmap : m.o, penmap ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_prefill_attention_tc(const CacheView& c, int T0, int T, void* o, const PrefillMaps& maps,
                                        cudaStream_t s, const float* pen, const CUtensorMap* penmap) {
  return c.D == 64 ? launch_tc<64>(c, T0, T, o, maps, s, pen, penmap)
                   : launch_tc<128>(c, T0, T, o, maps, s, pen, penmap);
}

// ---------------------------------------------------------------------------
// Gate of the training path, one thread per token: l = (alpha + noise) / tau,
// prob = sigmoid(l), hard = 1 if l > 0 else 0 (the forward value of the
// straight-through decision, prob > 0.5), and the penalty of the next
// position, logsigmoid(-l) (position 0 of each row gets 0).
// ---------------------------------------------------------------------------
__global__ void k_train_gate(long n, int T, const float* alpha, const float* noise, float tau, float* prob,
                             float* hard, float* penalty) {
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const float l = __fdiv_rn(alpha[i] + (noise ? noise[i] : 0.f), tau);
    prob[i] = 1.0f / (1.0f + expf(-l));
    hard[i] = l > 0.f ? 1.0f : 0.0f;
    // logsigmoid(-l) = -log(1 + exp(l)), without overflow for large l
    const float ls = l > 0.f ? -(l + log1pf(expf(-l))) : -log1pf(expf(l));
    const int t = static_cast<int>(i % T);
    if (t + 1 < T) penalty[i + 1] = ls;
    if (t == 0) penalty[i] = 0.f;
  }
}

cudaError_t launch_train_gate(long rows, int T, const float* alpha, const float* noise, float tau, float* prob,
                              float* hard, float* penalty, int num_sms, cudaStream_t s) {
  const long n = rows * T;
  const int grid = static_cast<int>(max(1L, min((n + 255) / 256, static_cast<long>(num_sms) * 8)));
  k_train_gate<<<grid, 256, 0, s>>>(n, T, alpha, noise, tau, prob, hard, penalty);
  return cudaGetLastError();
}

}  // namespace dms

