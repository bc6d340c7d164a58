// Device building blocks shared by the decode attention kernels.
#pragma once

#include "dms_internal.cuh"

namespace dms {

constexpr int kSub = 64;     // slots per sub-tile
constexpr int kStages = 3;   // shared-memory stages of the TMA ring
constexpr int kThreads = 128;

template <int D, bool FP8>
struct DecodeSmem {
  static constexpr int HALVES = D / 64;                 // 128-byte column halves of a bf16 row
  static constexpr int TILE_BF16 = kSub * D * 2;        // bytes of one bf16 K (or V) sub-tile
  static constexpr int TILE_RAW = FP8 ? kSub * D : TILE_BF16;
  static constexpr int STAGE = 2 * TILE_RAW;            // K then V, as loaded
  static constexpr int CONV = FP8 ? 2 * TILE_BF16 : 0;  // widened bf16 K and V (FP8 only)
};

struct StageMeta {
  int item;  // work item index
  int bh;    // (b, h) of the item
  int s0;    // first slot of the item
  int sub;   // first slot of the sub-tile, relative to the item start
  int rows;  // valid slots in the sub-tile
  int page;  // page id
  int last;  // 1 if this is the item's last sub-tile
};

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a tile written
// by TMA with the 128-byte swizzle (1024-byte aligned tile).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Issue the TMA loads of one sub-tile (`rows` slots starting at pool row
// `row0`, all inside one page) into a stage: K then V, 16-row boxes; bf16 rows
// as 128-byte column halves with the 128-byte swizzle, FP8 rows unswizzled.
// Called by one thread; completes on `bar` with the exact byte count.
template <int D, bool FP8>
__device__ __forceinline__ void issue_subtile(unsigned char* dst, const CUtensorMap* kmap, const CUtensorMap* vmap,
                                              int row0, int rows, uint64_t* bar) {
  using S = DecodeSmem<D, FP8>;
  const int nbox = (rows + 15) / 16;
  const uint32_t bytes = static_cast<uint32_t>(nbox * 16 * (FP8 ? D : 128) * (FP8 ? 1 : S::HALVES) * 2);
  mbar_expect_tx(bar, bytes);
  for (int bx = 0; bx < nbox; ++bx) {
    if (FP8) {
      tma_load_2d(dst + bx * 16 * D, kmap, 0, row0 + bx * 16, bar);
      tma_load_2d(dst + S::TILE_RAW + bx * 16 * D, vmap, 0, row0 + bx * 16, bar);
    } else {
      for (int hf = 0; hf < S::HALVES; ++hf) {
        tma_load_2d(dst + hf * kSub * 128 + bx * 16 * 128, kmap, hf * 64, row0 + bx * 16, bar);
        tma_load_2d(dst + S::TILE_RAW + hf * kSub * 128 + bx * 16 * 128, vmap, hf * 64, row0 + bx * 16, bar);
      }
    }
  }
}

// Issue the TMA loads of `rows` slots (<= TROWS, starting at pool row `row0`,
// all inside one page) into a stage of TROWS-row tiles: K then V, 16-row
// boxes; bf16 rows as 128-byte column halves with the 128-byte swizzle (half
// hf at hf * TROWS * 128), FP8 rows unswizzled.  Called by one thread;
// completes on `bar` with the exact byte count.
template <int D, bool FP8, int TROWS>
__device__ __forceinline__ void issue_rows(unsigned char* dst, const CUtensorMap* kmap, const CUtensorMap* vmap,
                                           int row0, int rows, uint64_t* bar) {
  constexpr int HALVES = D / 64, TILE = FP8 ? TROWS * D : TROWS * D * 2;
  const int nbox = (rows + 15) / 16;
  mbar_expect_tx(bar, static_cast<uint32_t>(nbox * 16 * D * (FP8 ? 1 : 2) * 2));
  for (int bx = 0; bx < nbox; ++bx) {
    if (FP8) {
      tma_load_2d(dst + bx * 16 * D, kmap, 0, row0 + bx * 16, bar);
      tma_load_2d(dst + TILE + bx * 16 * D, vmap, 0, row0 + bx * 16, bar);
    } else {
#pragma unroll
      for (int hf = 0; hf < HALVES; ++hf) {
        tma_load_2d(dst + hf * TROWS * 128 + bx * 16 * 128, kmap, hf * 64, row0 + bx * 16, bar);
        tma_load_2d(dst + TILE + hf * TROWS * 128 + bx * 16 * 128, vmap, hf * 64, row0 + bx * 16, bar);
      }
    }
  }
}

// 2-D TMA tile load (no multicast) with an L2 cache policy: the KV pages are
// read once per step, so they are marked first to evict, which keeps the
// small per-layer state (plans, page tables, ring) resident in L2 between
// the steps of a deep layer stack.
__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* map, int c0, int c1,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3}], [%4], %5;\n" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}

// Issue the TMA loads of one TROWS-row sub-tile starting at pool row `row0`
// into a stage: K then V, one TROWS-row box per 128-byte column half (bf16,
// 128-byte swizzle) or one box of 128-byte lines of codes (FP8, 128-byte
// swizzle; two rows per line for D = 64, row0 even); rows past the sub-tile's own
// are read along (pool rows, finite; the pool's end reads as zeros) and
// masked by the consumer.  Called by one thread; completes on `bar`.
template <int D, bool FP8, int TROWS>
__device__ __forceinline__ void issue_tile(unsigned char* dst, const CUtensorMap* kmap, const CUtensorMap* vmap,
                                           int row0, uint64_t* bar, uint64_t policy) {
  constexpr int HALVES = D / 64, TILE = FP8 ? TROWS * D : TROWS * D * 2;
  mbar_expect_tx(bar, static_cast<uint32_t>(2 * TILE));
  if (FP8) {
    // (64-code rows: the maps' lines hold two rows; row0 is even)
    const int line0 = D == 64 ? row0 >> 1 : row0;
    tma_load_2d_hint(dst, kmap, 0, line0, bar, policy);
    tma_load_2d_hint(dst + TILE, vmap, 0, line0, bar, policy);
  } else {
#pragma unroll
    for (int hf = 0; hf < HALVES; ++hf) {
      tma_load_2d_hint(dst + hf * TROWS * 128, kmap, hf * 64, row0, bar, policy);
      tma_load_2d_hint(dst + TILE + hf * TROWS * 128, vmap, hf * 64, row0, bar, policy);
    }
  }
}

// Widen a staged FP8 sub-tile (K then V, unswizzled rows of D codes) to bf16
// codes (exact) in the 128-byte swizzled layout of `conv` (K then V).
template <int D>
__device__ __forceinline__ void widen_fp8_subtile(const unsigned char* raw, unsigned char* conv) {
  constexpr int TILE_RAW = kSub * D, TILE_BF16 = kSub * D * 2, CH = D / 16;
  for (int idx = threadIdx.x; idx < 2 * kSub * CH; idx += kThreads) {
    const int which = idx / (kSub * CH);
    const int rem = idx % (kSub * CH);
    const int r = rem / CH, ch = rem % CH;  // 16 codes
    const uint4 u = *reinterpret_cast<const uint4*>(raw + which * TILE_RAW + r * D + ch * 16);
    const uint8_t* cb = reinterpret_cast<const uint8_t*>(&u);
    uint32_t wds[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) wds[e] = pack_bf16(fp8_decode(cb[2 * e]), fp8_decode(cb[2 * e + 1]));
    unsigned char* dstt = conv + which * TILE_BF16;
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const int chunk = 2 * ch + hc;
      *reinterpret_cast<uint4*>(dstt + (chunk / 8) * kSub * 128 + sw128(r, chunk % 8)) =
          make_uint4(wds[4 * hc], wds[4 * hc + 1], wds[4 * hc + 2], wds[4 * hc + 3]);
    }
  }
}

// Per-CTA work partition of one layer's decode attention, identical in every
// CTA: chunk C = the largest power-of-two divisor of P (>= 16) giving at least
// `target` items; item j of head bh covers slots [j*C, min(count, (j+1)*C)),
// which lie in one page.  s_cnt[BH] and s_off[BH + 1] are shared memory;
// `red` holds 32 x 4 ints.  Returns C; s_off[BH] is the item count.
__device__ __forceinline__ int decode_partition(const int* count, int BH, int P, int target, int* s_cnt, int* s_off,
                                                int (*red)[4]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int part[4] = {0, 0, 0, 0};
  for (int i = tid; i < BH; i += kThreads) {
    const int cnt = count[i];
    s_cnt[i] = cnt;
#pragma unroll
    for (int k = 0; k < 4; ++k) part[k] += (cnt + (P >> k) - 1) / (P >> k);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part[k] += __shfl_xor_sync(0xffffffffu, part[k], o);
  __syncthreads();
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < 4; ++k) red[warp][k] = part[k];
  __syncthreads();
  int C = P;
  for (int k = 0; k < 4; ++k) {
    C = P >> k;
    const int tot = red[0][k] + red[1][k] + red[2][k] + red[3][k];
    const int next = C / 2;
    if (tot >= target || next % 16 != 0 || P % next != 0) break;
  }
  __syncthreads();
  int base = 0;
  for (int i0 = 0; i0 < BH; i0 += kThreads) {
    const int i = i0 + tid;
    const int n = i < BH ? (s_cnt[i] + C - 1) / C : 0;
    int tot;
    const int off = block_exclusive_scan(n, &red[0][0], &tot);
    if (i < BH) s_off[i] = base + off;
    base += tot;
  }
  if (tid == 0) s_off[BH] = base;
  __syncthreads();
  return C;
}

// Q fragments (mma.sync A operand) of the g query heads sharing a KV head;
// rows >= g are zero.
template <int D>
__device__ __forceinline__ void load_q_frags(const __nv_bfloat16* qb, int g, uint32_t (&qa)[D / 16][4]) {
  const int lane = threadIdx.x & 31;
  const int ra = lane >> 2, rb = ra + 8;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int col = ks * 16 + 2 * (lane & 3);
    qa[ks][0] = ra < g ? *reinterpret_cast<const uint32_t*>(qb + static_cast<long>(ra) * D + col) : 0u;
    qa[ks][1] = rb < g ? *reinterpret_cast<const uint32_t*>(qb + static_cast<long>(rb) * D + col) : 0u;
    qa[ks][2] = ra < g ? *reinterpret_cast<const uint32_t*>(qb + static_cast<long>(ra) * D + col + 8) : 0u;
    qa[ks][3] = rb < g ? *reinterpret_cast<const uint32_t*>(qb + static_cast<long>(rb) * D + col + 8) : 0u;
  }
}

// One warp's online-softmax update over keys warp*16 .. warp*16+15 of a
// staged sub-tile (bf16, 128-byte swizzled, column halves of 64 elements).
// Keys >= rows and key `masked` are excluded.  Scores are in the log2 domain:
// s = q.k * kscale * log2(e) / sqrt(D).  The probabilities entering PV are
// multiplied by `vscale` (the FP8 page scale of V; 1 for bf16 pages), the row
// sums are not.
template <int D>
__device__ __forceinline__ void warp_tile(const unsigned char* kt, const unsigned char* vt, int rows, int masked,
                                          float kscale_l2, float vscale, const uint32_t (&qa)[D / 16][4],
                                          float (&acc)[D / 8][4], float (&mrow)[2], float (&lrow)[2]) {
  constexpr int KS = D / 16, NT = D / 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int mi = lane >> 3, rr = lane & 7;
  float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int n_row = warp * 16 + (mi >> 1) * 8 + rr;
    const int chunk = 2 * ks + (mi & 1);
    uint32_t b0, b1, b2, b3;
    ldmatrix_x4(b0, b1, b2, b3, smem_u32(kt + (chunk / 8) * kSub * 128 + sw128(n_row, chunk % 8)));
    uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
    mma_bf16_16816(s[0], qa[ks], bb0);
    mma_bf16_16816(s[1], qa[ks], bb1);
  }
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = warp * 16 + nt * 8 + 2 * (lane & 3) + (e & 1);
      const float x = (key < rows && key != masked) ? s[nt][e] * kscale_l2 : -INFINITY;
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
  pa[0] = pack_bf16(s[0][0] * vscale, s[0][1] * vscale);
  pa[1] = pack_bf16(s[0][2] * vscale, s[0][3] * vscale);
  pa[2] = pack_bf16(s[1][0] * vscale, s[1][1] * vscale);
  pa[3] = pack_bf16(s[1][2] * vscale, s[1][3] * vscale);
#pragma unroll
  for (int dp = 0; dp < NT / 2; ++dp) {
    const int n_row = warp * 16 + (mi & 1) * 8 + rr;
    const int chunk = 2 * dp + (mi >> 1);
    uint32_t b0, b1, b2, b3;
    ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(vt + (chunk / 8) * kSub * 128 + sw128(n_row, chunk % 8)));
    uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
    mma_bf16_16816(acc[2 * dp], pa, bb0);
    mma_bf16_16816(acc[2 * dp + 1], pa, bb1);
  }
}

// One warp's online-softmax update over KEYS consecutive keys of a staged tile
// (bf16, 128-byte swizzled, column halves of TROWS rows of 128 bytes; K and V
// alike), keys numbered from 0 at the tile's first row.  Keys >= rows and key
// `masked` are excluded.  Scores are in the log2 domain: s = q.k * kscale *
// log2(e) / sqrt(D).  The probabilities entering PV are multiplied by `vscale`
// (the FP8 page scale of V; 1 for bf16 pages), the row sums are not.  The
// QK^T products of the KEYS/16 key pairs and the PV products of the D/16
// column pairs are independent mma chains, so one warp keeps the tensor pipe
// busy on its own.
template <int D, int KEYS, int TROWS>
__device__ __forceinline__ void warp_tile_keys(const unsigned char* kt, const unsigned char* vt, int rows, int masked,
                                               float kscale_l2, float vscale, const uint32_t (&qa)[D / 16][4],
                                               float (&acc)[D / 8][4], float (&mrow)[2], float (&lrow)[2]) {
  constexpr int KS = D / 16, NT = D / 8, KP = KEYS / 16;
  const int lane = threadIdx.x & 31;
  const int mi = lane >> 3, rr = lane & 7;
  float s[KP][2][4];
#pragma unroll
  for (int kp = 0; kp < KP; ++kp)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) s[kp][nt][0] = s[kp][nt][1] = s[kp][nt][2] = s[kp][nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int chunk = 2 * ks + (mi & 1);
#pragma unroll
    for (int kp = 0; kp < KP; ++kp) {
      const int n_row = kp * 16 + (mi >> 1) * 8 + rr;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(b0, b1, b2, b3, smem_u32(kt + (chunk / 8) * TROWS * 128 + sw128(n_row, chunk % 8)));
      uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
      mma_bf16_16816(s[kp][0], qa[ks], bb0);
      mma_bf16_16816(s[kp][1], qa[ks], bb1);
    }
  }
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int kp = 0; kp < KP; ++kp)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kp * 16 + nt * 8 + 2 * (lane & 3) + (e & 1);
        const float x = (key < rows && key != masked) ? s[kp][nt][e] * kscale_l2 : -INFINITY;
        s[kp][nt][e] = x;
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
  for (int kp = 0; kp < KP; ++kp)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[kp][nt][e] - mu[e >> 1]);
        s[kp][nt][e] = p;
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
#pragma unroll
  for (int kp = 0; kp < KP; ++kp) {
    uint32_t pa[4];
    pa[0] = pack_bf16(s[kp][0][0] * vscale, s[kp][0][1] * vscale);
    pa[1] = pack_bf16(s[kp][0][2] * vscale, s[kp][0][3] * vscale);
    pa[2] = pack_bf16(s[kp][1][0] * vscale, s[kp][1][1] * vscale);
    pa[3] = pack_bf16(s[kp][1][2] * vscale, s[kp][1][3] * vscale);
    const int n_row = kp * 16 + (mi & 1) * 8 + rr;
#pragma unroll
    for (int dp = 0; dp < NT / 2; ++dp) {
      const int chunk = 2 * dp + (mi >> 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(vt + (chunk / 8) * TROWS * 128 + sw128(n_row, chunk % 8)));
      uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
      mma_bf16_16816(acc[2 * dp], pa, bb0);
      mma_bf16_16816(acc[2 * dp + 1], pa, bb1);
    }
  }
}

// Widen rows [r0, r0 + CROWS) of a staged FP8 sub-tile (K then V, RAWROWS
// unswizzled rows of D codes each) to bf16 (exact) in the 128-byte swizzled
// layout of a CROWS-row tile pair at `conv` (K then V), by one warp.
template <int D, int CROWS, int RAWROWS>
__device__ __forceinline__ void widen_fp8_rows(const unsigned char* raw, unsigned char* conv, int r0) {
  constexpr int TILE_RAW = RAWROWS * D, CTILE = CROWS * D * 2, CH = D / 16;
  const int lane = threadIdx.x & 31;
  for (int idx = lane; idx < 2 * CROWS * CH; idx += 32) {
    const int which = idx / (CROWS * CH);
    const int rem = idx % (CROWS * CH);
    const int r = rem / CH, ch = rem % CH;  // 16 codes of row r0 + r
    const uint4 u = *reinterpret_cast<const uint4*>(raw + which * TILE_RAW + (r0 + r) * D + ch * 16);
    const uint32_t wsrc[4] = {u.x, u.y, u.z, u.w};
    uint32_t wds[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half2_raw lo =
          __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(wsrc[e] & 0xFFFFu), __NV_E4M3);
      const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(wsrc[e] >> 16), __NV_E4M3);
      const float2 fl = __half22float2(__half2(lo)), fh = __half22float2(__half2(hi));
      wds[2 * e] = pack_bf16(fl.x, fl.y);
      wds[2 * e + 1] = pack_bf16(fh.x, fh.y);
    }
    unsigned char* dstt = conv + which * CTILE;
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const int chunk = 2 * ch + hc;
      *reinterpret_cast<uint4*>(dstt + (chunk / 8) * CROWS * 128 + sw128(r, chunk % 8)) =
          make_uint4(wds[4 * hc], wds[4 * hc + 1], wds[4 * hc + 2], wds[4 * hc + 3]);
    }
  }
}

// 8x8 bf16 matrix transpose across the warp (the mma fragment layout: lane
// holds row lane / 4, columns 2 (lane % 4) + {0, 1}).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// warp_tile_keys with the keys as the M dimension of the mma tiles and the
// g <= 8 query heads as N = 8: S^T = K Q^T, then O^T += V^T P^T.  For g <= 8
// this takes half the tensor work of the query-major form (whose M = 16 rows
// hold only g queries).  Lane state: queries 2 (lane % 4) + {0, 1}; running
// maxima uniform over the lanes sharing lane % 4, sums partial per lane.
//   qb[ks]: Q as the B operand: Q[lane / 4][16 ks + 2 (lane % 4) + {0, 1}]
//           and the same + 8 (rows >= g zero).
//   acc[dt][j], acc[dt][2 + j]: O^T[16 dt + lane / 4 (+ 8)][2 (lane % 4) + j].
// The probability tiles go from the S^T accumulator layout to the B operand
// of the PV product by an in-register 8x8 transpose (movmatrix).
template <int D, int KEYS, int TROWS>
__device__ __forceinline__ void warp_tile_keys_t(const unsigned char* kt, const unsigned char* vt, int rows,
                                                 int masked, float kscale_l2, float vscale,
                                                 const uint32_t (&qb)[D / 16][2], float (&acc)[D / 16][4],
                                                 float (&mrow)[2], float (&lrow)[2]) {
  constexpr int KS = D / 16, MT = KEYS / 16, DT = D / 16;
  const int lane = threadIdx.x & 31;
  float s[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int chunk = 2 * ks + (lane >> 4);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      uint32_t a[4];
      ldmatrix_x4(a[0], a[1], a[2], a[3],
                  smem_u32(kt + (chunk / 8) * TROWS * 128 + sw128(mt * 16 + (lane & 15), chunk % 8)));
      mma_bf16_16816(s[mt], a, qb[ks]);
    }
  }
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = mt * 16 + (lane >> 2) + (e >> 1) * 8;
      const float x = (key < rows && key != masked) ? s[mt][e] * kscale_l2 : -INFINITY;
      s[mt][e] = x;
      mx[e & 1] = fmaxf(mx[e & 1], x);
    }
  float corr[2], mu[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 4));
    mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 8));
    mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 16));
    const float mn = fmaxf(mrow[j], mx[j]);
    mu[j] = mn == -INFINITY ? 0.f : mn;
    corr[j] = exp2f(mrow[j] - mu[j]);
    mrow[j] = mn;
  }
  float rs[2] = {0.f, 0.f};
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float p = exp2f(s[mt][e] - mu[e & 1]);
      s[mt][e] = p;
      rs[e & 1] += p;
    }
  lrow[0] = lrow[0] * corr[0] + rs[0];
  lrow[1] = lrow[1] * corr[1] + rs[1];
#pragma unroll
  for (int dt = 0; dt < DT; ++dt) {
    acc[dt][0] *= corr[0];
    acc[dt][1] *= corr[1];
    acc[dt][2] *= corr[0];
    acc[dt][3] *= corr[1];
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    uint32_t pb[2];
    pb[0] = movmatrix_trans(pack_bf16(s[mt][0] * vscale, s[mt][1] * vscale));  // keys 16 mt + 0..7
    pb[1] = movmatrix_trans(pack_bf16(s[mt][2] * vscale, s[mt][3] * vscale));  // keys 16 mt + 8..15
    const int key = mt * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
    for (int dt = 0; dt < DT; ++dt) {
      const int chunk = 2 * dt + ((lane >> 3) & 1);
      uint32_t a[4];
      ldmatrix_x4_trans(a[0], a[1], a[2], a[3], smem_u32(vt + (chunk / 8) * TROWS * 128 + sw128(key, chunk % 8)));
      mma_bf16_16816(acc[dt], a, pb);
    }
  }
}

// ---- FP8 pages on f16 tensor cores --------------------------------------
// E4M3 codes convert exactly to f16, two per instruction.  FP8 tiles are
// staged by TMA as 128-byte lines with the 128-byte swizzle (16-byte chunk c
// of line l at c ^ (l & 7)): a line is one row of 128 codes, or, for D = 64,
// two consecutive rows (so that every request TMA makes is 128 bytes), and
// eight rows' same chunk fall in different banks.
template <int D>
__device__ __forceinline__ int fp8_sw_off(int row, int chunk) {
  if (D == 128) return row * 128 + ((chunk ^ (row & 7)) << 4);
  const int line = row >> 1;
  return line * 128 + ((((row & 1) << 2 | chunk) ^ (line & 7)) << 4);
}
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xFFFFu), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// D = A * B + D, m16n8k16, f16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_f16_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Widen ROWS rows of a staged, swizzled FP8 tile (D codes per row) to 16-bit
// values (f16 when F16, else bf16; both exact) in the 128-byte swizzled layout
// of a ROWS-row tile (column halves of 64 elements), by one warp.
template <int D, int ROWS, bool F16>
__device__ __forceinline__ void widen_fp8_tile(const unsigned char* raw, unsigned char* conv) {
  constexpr int CH = D / 16;
  const int lane = threadIdx.x & 31;
  for (int idx = lane; idx < ROWS * CH; idx += 32) {
    const int r = idx / CH, ch = idx % CH;  // 16 codes of row r
    const uint4 u = *reinterpret_cast<const uint4*>(raw + fp8_sw_off<D>(r, ch));
    const uint32_t wsrc[4] = {u.x, u.y, u.z, u.w};
    uint32_t wds[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = e4m3x2_to_f16x2(wsrc[e]), hi = e4m3x2_to_f16x2(wsrc[e] >> 16);
      if (F16) {
        wds[2 * e] = lo;
        wds[2 * e + 1] = hi;
      } else {
        const float2 fl = __half22float2(*reinterpret_cast<const __half2*>(&lo));
        const float2 fh = __half22float2(*reinterpret_cast<const __half2*>(&hi));
        wds[2 * e] = pack_bf16(fl.x, fl.y);
        wds[2 * e + 1] = pack_bf16(fh.x, fh.y);
      }
    }
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const int chunk = 2 * ch + hc;
      *reinterpret_cast<uint4*>(conv + (chunk / 8) * ROWS * 128 + sw128(r, chunk % 8)) =
          make_uint4(wds[4 * hc], wds[4 * hc + 1], wds[4 * hc + 2], wds[4 * hc + 3]);
    }
  }
}

// Query rows as f16 B operands of warp_tile_keys_fp8: qh[ks] = Q[lane / 4]
// [16 ks + 4 (lane % 4) + {0, 1}] and [... + {2, 3}] (rows >= g zero) -- the
// k order of the K fragments that ldmatrix gives on raw FP8 rows.
template <int D>
__device__ __forceinline__ void load_q_frags_fp8(const __nv_bfloat16* qb, int g, uint32_t (&qh)[D / 16][2]) {
  const int lane = threadIdx.x & 31, r = lane >> 2, j = lane & 3;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    if (r < g) {
      const uint2 u = *reinterpret_cast<const uint2*>(qb + static_cast<long>(r) * D + 16 * ks + 4 * j);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
      qh[ks][0] = pack_f16(a.x, a.y);
      qh[ks][1] = pack_f16(b.x, b.y);
    } else {
      qh[ks][0] = qh[ks][1] = 0u;
    }
  }
}

// warp_tile_keys_t for FP8 pages: S^T = K Q^T with the K fragments taken by
// ldmatrix straight from the swizzled FP8 rows and converted in registers
// (lane's word of an 8x8 matrix is 4 codes, k slots 2j + e and 8 + 2j + e
// holding codes 4j + e and 4j + 2 + e, j = lane % 4; qh follows the same
// order), then O^T += V^T P^T from V widened to f16 (vt: a ROWS-row tile in
// the 128-byte swizzled layout).  Scores in the log2 domain with the page's
// K scale in kscale_l2; P carries the V scale.
template <int D, int KEYS, int TROWS>
__device__ __forceinline__ void warp_tile_keys_fp8(const unsigned char* kraw, const unsigned char* vt, int rows,
                                                   int masked, float kscale_l2, float vscale,
                                                   const uint32_t (&qh)[D / 16][2], float (&acc)[D / 16][4],
                                                   float (&mrow)[2], float (&lrow)[2]) {
  constexpr int MT = KEYS / 16, DT = D / 16;
  const int lane = threadIdx.x & 31;
  float s[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
#pragma unroll
  for (int kp = 0; kp < D / 32; ++kp) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int i = lane >> 3;
      const int key = mt * 16 + (lane & 7) + (i & 1) * 8;
      uint32_t r0, r1, r2, r3;
      ldmatrix_x4(r0, r1, r2, r3, smem_u32(kraw + fp8_sw_off<D>(key, 2 * kp + (i >> 1))));
      const uint32_t a0[4] = {e4m3x2_to_f16x2(r0), e4m3x2_to_f16x2(r1), e4m3x2_to_f16x2(r0 >> 16),
                              e4m3x2_to_f16x2(r1 >> 16)};
      const uint32_t a1[4] = {e4m3x2_to_f16x2(r2), e4m3x2_to_f16x2(r3), e4m3x2_to_f16x2(r2 >> 16),
                              e4m3x2_to_f16x2(r3 >> 16)};
      mma_f16_16816(s[mt], a0, qh[2 * kp]);
      mma_f16_16816(s[mt], a1, qh[2 * kp + 1]);
    }
  }
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = mt * 16 + (lane >> 2) + (e >> 1) * 8;
      const float x = (key < rows && key != masked) ? s[mt][e] * kscale_l2 : -INFINITY;
      s[mt][e] = x;
      mx[e & 1] = fmaxf(mx[e & 1], x);
    }
  float corr[2], mu[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 4));
    mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 8));
    mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 16));
    const float mn = fmaxf(mrow[j], mx[j]);
    mu[j] = mn == -INFINITY ? 0.f : mn;
    corr[j] = exp2f(mrow[j] - mu[j]);
    mrow[j] = mn;
  }
  float rs[2] = {0.f, 0.f};
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float p = exp2f(s[mt][e] - mu[e & 1]);
      s[mt][e] = p;
      rs[e & 1] += p;
    }
  lrow[0] = lrow[0] * corr[0] + rs[0];
  lrow[1] = lrow[1] * corr[1] + rs[1];
#pragma unroll
  for (int dt = 0; dt < DT; ++dt) {
    acc[dt][0] *= corr[0];
    acc[dt][1] *= corr[1];
    acc[dt][2] *= corr[0];
    acc[dt][3] *= corr[1];
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    uint32_t pb[2];
    pb[0] = movmatrix_trans(pack_f16(s[mt][0] * vscale, s[mt][1] * vscale));
    pb[1] = movmatrix_trans(pack_f16(s[mt][2] * vscale, s[mt][3] * vscale));
    const int key = mt * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
    for (int dt = 0; dt < DT; ++dt) {
      const int chunk = 2 * dt + ((lane >> 3) & 1);
      uint32_t a[4];
      ldmatrix_x4_trans(a[0], a[1], a[2], a[3], smem_u32(vt + (chunk / 8) * TROWS * 128 + sw128(key, chunk % 8)));
      mma_f16_16816(acc[dt], a, pb);
    }
  }
}

// The state of warp_tile_keys_t (queries < g) into merge buffer slot `src`,
// laid out as warp_state_to_smem's.
template <int D>
__device__ __forceinline__ void warp_state_t_to_smem(float* merge, int src, int g, const float (&acc)[D / 16][4],
                                                     const float (&mrow)[2], const float (&lrow)[2]) {
  constexpr int DT = D / 16, MLD = D + 2;
  const int lane = threadIdx.x & 31;
  float lsum[2] = {lrow[0], lrow[1]};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    lsum[j] += __shfl_xor_sync(0xffffffffu, lsum[j], 4);
    lsum[j] += __shfl_xor_sync(0xffffffffu, lsum[j], 8);
    lsum[j] += __shfl_xor_sync(0xffffffffu, lsum[j], 16);
  }
  float* mw = merge + src * g * MLD;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int qr = 2 * (lane & 3) + j;
    if (qr < g) {
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        mw[qr * MLD + dt * 16 + (lane >> 2)] = acc[dt][j];
        mw[qr * MLD + dt * 16 + (lane >> 2) + 8] = acc[dt][2 + j];
      }
      if (lane < 4) {
        mw[qr * MLD + D] = mrow[j];
        mw[qr * MLD + D + 1] = lsum[j];
      }
    }
  }
}

// Store one warp's state (rows < g) into the merge buffer slot `src`:
// merge[(src * g + r) * (D + 2) + {0..D-1: acc, D: max, D+1: sum}].
template <int D>
__device__ __forceinline__ void warp_state_to_smem(float* merge, int src, int g, const float (&acc)[D / 8][4],
                                                   const float (&mrow)[2], const float (&lrow)[2]) {
  constexpr int NT = D / 8, MLD = D + 2;
  const int lane = threadIdx.x & 31;
  const int ra = lane >> 2, rb = ra + 8;
  float lsum[2] = {lrow[0], lrow[1]};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lsum[r] += __shfl_xor_sync(0xffffffffu, lsum[r], 1);
    lsum[r] += __shfl_xor_sync(0xffffffffu, lsum[r], 2);
  }
  float* mw = merge + src * g * MLD;
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
}

// Merge `nsrc` staged states per row into (acc scaled by vscale, running max,
// running sum) and hand each value to store(r, d, value) with d in [0, D + 1]
// (d == D: the max, d == D + 1: the sum).
template <int D, typename Store>
__device__ __forceinline__ void merge_sources(const float* merge, int nsrc, int g, float vscale, Store store) {
  constexpr int MLD = D + 2;
  for (int idx = threadIdx.x; idx < g * (D + 1); idx += kThreads) {
    const int r = idx / (D + 1), d = idx % (D + 1);
    float M = -INFINITY;
    for (int sv = 0; sv < nsrc; ++sv) M = fmaxf(M, merge[(sv * g + r) * MLD + D]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float sum = 0.f;
    for (int sv = 0; sv < nsrc; ++sv) {
      const float f = exp2f(merge[(sv * g + r) * MLD + D] - Mu);
      sum += f * merge[(sv * g + r) * MLD + (d < D ? d : D + 1)];
    }
    if (d < D) {
      store(r, d, sum * vscale);
    } else {
      store(r, D, M);
      store(r, D + 1, sum);
    }
  }
}

// ... into an item's partial in global scratch.
template <int D>
__device__ __forceinline__ void merge_to_global(const float* merge, int nsrc, int g, float vscale, float* part_acc,
                                                float* part_ml, long item) {
  merge_sources<D>(merge, nsrc, g, vscale, [&](int r, int d, float v) {
    if (d < D)
      part_acc[(item * g + r) * D + d] = v;
    else
      part_ml[(item * g + r) * 2 + (d - D)] = v;
  });
}

// LSE combine of a head's partials (items i0..i1) by one CTA:
//   o[r] = sum_i 2^(m_i[r] - M[r]) acc_i[r] / sum_i 2^(m_i[r] - M[r]) l_i[r].
// The maxima and weights are staged in shared memory (`wbuf`, at least
// 2 * kCombineChunk + 16 floats), then each thread owns 4 consecutive output
// columns of one row and issues its 16-byte loads for all items of a chunk
// before using them, so the merge costs a few L2 round trips.
constexpr int kCombineChunk = 256;  // (item, row) pairs staged per pass

template <int D>
__device__ void combine_head(const float* part_acc, const float* part_ml, int g, int i0, int i1,
                             __nv_bfloat16* out /* [g, D] rows of this head */, float* wbuf) {
  const int tid = threadIdx.x;
  float* s_M = wbuf + 2 * kCombineChunk;  // [g <= 16]
  float* s_L = s_M + 16;                 // [g]  (wbuf holds 2*kCombineChunk + 32 floats)
  if (tid < g) {
    s_M[tid] = -INFINITY;
    s_L[tid] = 0.f;
  }
  constexpr int Q = D / 4;                            // float4 columns per row
  constexpr int OUTS = (16 * Q + kThreads - 1) / kThreads;  // float4 outputs per thread (g <= 16)
  float4 accv[OUTS];
#pragma unroll
  for (int k = 0; k < OUTS; ++k) accv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int per_chunk = max(1, kCombineChunk / g);
  for (int c0 = i0; c0 < i1; c0 += per_chunk) {
    const int n = min(i1, c0 + per_chunk) - c0;
    __syncthreads();
    for (int idx = tid; idx < n * g; idx += kThreads) {
      const long e = (static_cast<long>(c0) * g + idx) * 2;
      wbuf[idx] = __ldcg(&part_ml[e]);
      wbuf[kCombineChunk + idx] = __ldcg(&part_ml[e + 1]);
    }
    __syncthreads();
    if (tid < g) {
      float M = s_M[tid];
      for (int i = 0; i < n; ++i) M = fmaxf(M, wbuf[i * g + tid]);
      const float Mu = M == -INFINITY ? 0.f : M;
      const float rescale = exp2f(s_M[tid] - Mu);
      float L = s_L[tid] * rescale;
      for (int i = 0; i < n; ++i) {
        const float wgt = exp2f(wbuf[i * g + tid] - Mu);
        wbuf[i * g + tid] = wgt;
        L += wgt * wbuf[kCombineChunk + i * g + tid];
      }
      wbuf[kCombineChunk + tid] = rescale;  // the sums are consumed; reuse the slot
      s_M[tid] = M;
      s_L[tid] = L;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < OUTS; ++k) {
      const int idx = tid + kThreads * k;
      if (idx >= g * Q) break;
      const int r = idx / Q, d4 = idx % Q;
      const float sc = wbuf[kCombineChunk + r];
      float4 a = accv[k];
      a.x *= sc;
      a.y *= sc;
      a.z *= sc;
      a.w *= sc;
      const float4* src = reinterpret_cast<const float4*>(part_acc) + (static_cast<long>(c0) * g + r) * Q + d4;
      const long stride = static_cast<long>(g) * Q;
      int i = 0;
      for (; i + 8 <= n; i += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (i + u) * stride);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float wgt = wbuf[(i + u) * g + r];
          a.x = fmaf(wgt, v[u].x, a.x);
          a.y = fmaf(wgt, v[u].y, a.y);
          a.z = fmaf(wgt, v[u].z, a.z);
          a.w = fmaf(wgt, v[u].w, a.w);
        }
      }
      for (; i < n; ++i) {
        const float4 v = __ldcg(src + i * stride);
        const float wgt = wbuf[i * g + r];
        a.x = fmaf(wgt, v.x, a.x);
        a.y = fmaf(wgt, v.y, a.y);
        a.z = fmaf(wgt, v.z, a.z);
        a.w = fmaf(wgt, v.w, a.w);
      }
      accv[k] = a;
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < OUTS; ++k) {
    const int idx = tid + kThreads * k;
    if (idx >= g * Q) break;
    const int r = idx / Q, d4 = idx % Q;
    const float L = s_L[r];
    const float inv = L > 0.f ? 1.f / L : 0.f;
    uint2 pk;
    pk.x = pack_bf16(accv[k].x * inv, accv[k].y * inv);
    pk.y = pack_bf16(accv[k].z * inv, accv[k].w * inv);
    *reinterpret_cast<uint2*>(out + static_cast<long>(r) * D + d4 * 4) = pk;
  }
}

// The decision logit of one (b, head) in pieces, so that its loads join the
// other loads of a prologue and its dot products can be shared by several
// CTAs: decide_issue starts the loads of part `part` of `nparts` equal slices
// of the hidden row (each at most kThreads * VPT 16-byte vectors; thread `who`
// also loads the bias and offset), decide_partial gives one thread's sums
// (x.x, (W * gamma).x), decide_reduce finishes a whole row in one CTA.
template <int VPT>
struct DecideLoads {
  uint4 x[VPT], w[VPT], gm[VPT];
  float bias, offset;
};
template <int VPT>
__device__ __forceinline__ void decide_issue(const CacheView& c, const DecideArgs& a, int b, int src,
                                             DecideLoads<VPT>& L, int part = 0, int nparts = 1, int who = 0) {
  const int tid = threadIdx.x, nvec = c.hidden / 8;
  const int per = (nvec + nparts - 1) / nparts, v0 = part * per, v1 = min(nvec, v0 + per);
  const uint4* xr =
      reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.hidden) + static_cast<long>(b) * c.hidden);
  const uint4* wr =
      reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.W) + static_cast<long>(src) * c.hidden);
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int vi = v0 + u * kThreads + tid;
    const bool ok = vi < v1;
    L.x[u] = ok ? xr[vi] : make_uint4(0, 0, 0, 0);
    L.w[u] = ok ? wr[vi] : make_uint4(0, 0, 0, 0);
    L.gm[u] = ok ? gamma16<__nv_bfloat16>(a.gamma, vi) : make_uint4(0, 0, 0, 0);
  }
  L.bias = 0.f;
  L.offset = 0.f;
  if (tid == who) {
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(a.bias);
    L.bias = bias ? __bfloat162float(bias[src]) : 0.f;
    L.offset = a.offset[b * a.offset_bstride + src];
  }
}
template <int VPT>
__device__ __forceinline__ float2 decide_partial(const DecideLoads<VPT>& L) {
  float ss = 0.f, dot = 0.f;
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    float x[8], wv[8], gv[8];
    unpack16(L.x[u], x, static_cast<const __nv_bfloat16*>(nullptr));
    unpack16(L.w[u], wv, static_cast<const __nv_bfloat16*>(nullptr));
    unpack16(L.gm[u], gv, static_cast<const __nv_bfloat16*>(nullptr));
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ss = fmaf(x[e], x[e], ss);
      dot = fmaf(wv[e] * gv[e], x[e], dot);
    }
  }
  return make_float2(ss, dot);
}
template <int VPT>
__device__ __forceinline__ float decide_reduce(const CacheView& c, const DecideLoads<VPT>& L, float* red) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const float2 pd = decide_partial<VPT>(L);
  float ss = pd.x, dot = pd.y;
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
  if (tid == 0)
    alpha = adapter_logit(c, red[4] + red[5] + red[6] + red[7], red[0] + red[1] + red[2] + red[3], c.hidden, L.bias,
                          L.offset);
  return alpha;
}

// Adapter decision logit of the new token of sequence b for head `src`, by one
// CTA of kThreads (all loads of a thread issued before use; bf16 operands).
// `red` holds 8 floats.  Returns the value in thread 0.
template <int VPT>
__device__ __forceinline__ float decide_cta(const CacheView& c, const DecideArgs& a, int b, int src, float* red) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int hid = c.hidden, nvec = hid / 8;
  const uint4* xr =
      reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.hidden) + static_cast<long>(b) * hid);
  const uint4* wr =
      reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.W) + static_cast<long>(src) * hid);
  float ss = 0.f, dot = 0.f;
  for (int v0 = 0; v0 < nvec; v0 += kThreads * VPT) {
    uint4 xu[VPT], wu[VPT], gu[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int vi = v0 + u * kThreads + tid;
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
    alpha = adapter_logit(c, d2, s2, hid, bias ? __bfloat162float(bias[src]) : 0.f, a.offset[b * a.offset_bstride + src]);
  }
  return alpha;
}

// Atomic add with acquire-release semantics at GPU scope (returns the old value).
__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// FP8 append of one token's K and V rows, each into a page of P rows of D
// codes with one scale per page ([DMS-Qwen3], FP8 KV pages): thread tid < D
// holds the rows' values kx = k[tid], vx = v[tid] (the others 0), and
// ks_old / vs_old are the pages' scales before the append.  When a row's
// amax / 448 exceeds its page's scale, the page's first `rows` rows are first
// re-encoded from their decoded values at the new scale (16 codes per thread
// and vector, four vectors in flight), and the scale is raised; then the row
// is encoded at row `r`.  Called by all kThreads threads of the block; `red`
// holds 2 * kThreads / 32 floats.  Returns the pages' scales after the append
// (in every thread).
__device__ __forceinline__ float2 fp8_append_kv(float kx, float vx, uint8_t* kpage, uint8_t* vpage, float* kscale_p,
                                               float* vscale_p, float ks_old, float vs_old, int r, int rows, int D,
                                               float* red) {
  constexpr int NW = kThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  float ka = fabsf(kx), va = fabsf(vx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ka = fmaxf(ka, __shfl_xor_sync(0xffffffffu, ka, o));
    va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, o));
  }
  if (lane == 0) {
    red[wid] = ka;
    red[NW + wid] = va;
  }
  __syncthreads();
  ka = va = 0.f;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    ka = fmaxf(ka, red[i]);
    va = fmaxf(va, red[NW + i]);
  }
  const float ks_new = __fdiv_rn(ka, 448.0f), vs_new = __fdiv_rn(va, 448.0f);
  const bool kgrow = ks_new > ks_old, vgrow = vs_new > vs_old;
  const int nvec = rows * D / 16;
  for (int which = 0; which < 2; ++which) {
    if (!(which ? vgrow : kgrow)) continue;
    const float s_old = which ? vs_old : ks_old, s_new = which ? vs_new : ks_new;
    uint4* pv = reinterpret_cast<uint4*>(which ? vpage : kpage);
    for (int v0 = 0; v0 < nvec; v0 += 4 * kThreads) {
      uint4 u[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int vi = v0 + e * kThreads + tid;
        if (vi < nvec) u[e] = pv[vi];
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int vi = v0 + e * kThreads + tid;
        if (vi >= nvec) continue;
        uint8_t* cb = reinterpret_cast<uint8_t*>(&u[e]);
#pragma unroll
        for (int j = 0; j < 16; ++j) cb[j] = fp8_encode(__fdiv_rn(__fmul_rn(fp8_decode(cb[j]), s_old), s_new));
        pv[vi] = u[e];
      }
    }
  }
  const float ks = kgrow ? ks_new : ks_old, vs = vgrow ? vs_new : vs_old;
  if (kgrow || vgrow) {
    __syncthreads();  // every code re-encoded before the rows and the scales
    if (tid == 0) {
      if (kgrow) *kscale_p = ks_new;
      if (vgrow) *vscale_p = vs_new;
    }
  }
  if (tid < D) {
    kpage[static_cast<long>(r) * D + tid] = ks > 0.f ? fp8_encode(__fdiv_rn(kx, ks)) : 0;
    vpage[static_cast<long>(r) * D + tid] = vs > 0.f ? fp8_encode(__fdiv_rn(vx, vs)) : 0;
  }
  __syncthreads();  // `red` reused by the caller
  return make_float2(ks, vs);
}

// Distributed shared memory (thread-block clusters).
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// The two halves of a cluster barrier: arrive without ordering this thread's
// memory operations (used right after the barrier initialisation, which its
// own fence releases), and wait (acquire).
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory"); }
// arrive releasing this thread's prior memory operations to the cluster
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
// this thread's prior generic-proxy writes to global memory, ordered before
// later async-proxy (TMA) accesses that synchronise with it
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
}
// Stores into another CTA's shared memory of the cluster that complete their
// bytes of the transaction count of an mbarrier there (16- and 8-byte aligned).
__device__ __forceinline__ void st_async_v4(uint32_t addr, float4 v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];\n" ::"r"(addr),
               "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)), "r"(__float_as_uint(v.z)), "r"(__float_as_uint(v.w)),
               "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t addr, float a, float b, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];\n" ::"r"(addr),
               "r"(__float_as_uint(a)), "r"(__float_as_uint(b)), "r"(bar)
               : "memory");
}
// 4-byte store of the same kind.
__device__ __forceinline__ void st_async_b32(uint32_t addr, float v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];\n" ::"r"(addr),
               "r"(__float_as_uint(v)), "r"(bar)
               : "memory");
}
// Address of `p` (this CTA's shared memory) in the shared memory of cluster rank `rank`.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_dsmem(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.b32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ float ld_dsmem(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Slot plan of the next append of head i of `layer` (token position t):
// reuse the slot of token t - w when it was marked for eviction, else take slot
// count (a new page when that slot starts one).  plan.x = slot,
// plan.y = bit 0 reuse | bit 1 new page | bit 2 over capacity; plan.z, plan.w =
// the head's retained count and pages before the append.
// Loads bypass L1: the state may have been written by other CTAs of the same
// launch (made visible by their fences).
// Step accounting of a fused decode launch: one 64-bit add per counting CTA,
// the CTAs arrived in the low word and the pages they granted in the high
// word, so the last CTA learns the step's total from its own add.  Every CTA
// has read the page counter and the positions before it counts itself, so
// the last one advances the counter (from next_page0, the value every CTA
// read) and the positions; what the other CTAs wrote is read only by later
// launches.  Returns true in the last CTA (thread that calls it).
__device__ __forceinline__ bool count_step(const CacheView& c, int granted, int ncount, int next_page0) {
  unsigned long long* done = reinterpret_cast<unsigned long long*>(&c.ctrl[CTRL_STEP64]);
  const unsigned long long mine = (static_cast<unsigned long long>(granted) << 32) | 1ull;
  const unsigned long long old = atomicAdd(done, mine);
  if (static_cast<int>(old & 0xffffffffull) != ncount - 1) return false;
  c.ctrl[CTRL_NEXT_PAGE] = min(next_page0 + static_cast<int>((old + mine) >> 32), c.pool_pages);
  *done = 0ull;
  return true;
}
__device__ __forceinline__ void advance_positions(const CacheView& c, int layer, int first, int stride, int nl = 1) {
  for (int bb = first; bb < nl * c.B; bb += stride) atomicAdd(&c.pos[layer * c.B + bb], 1);
}

__device__ __forceinline__ int4 make_plan(int ringv, int t, int cnt, int have, const CacheView& c) {
  if (t >= c.w && (static_cast<unsigned>(ringv) & RING_EVICT)) return make_int4(ringv & RING_SLOT_MASK, 1, cnt, have);
  if (cnt >= c.cap) return make_int4(-1, 4, cnt, have);
  return make_int4(cnt, (cnt % c.P == 0 && cnt / c.P >= have) ? 2 : 0, cnt, have);
}
__device__ __forceinline__ int4 next_plan(const CacheView& c, long li, int t) {
  const int cnt = __ldcg(&c.count[li]), have = __ldcg(&c.npages[li]);
  const int ringv = t >= c.w ? __ldcg(&c.ring[li * c.w + t % c.w]) : 0;
  return make_plan(ringv, t, cnt, have, c);
}

}  // namespace dms
