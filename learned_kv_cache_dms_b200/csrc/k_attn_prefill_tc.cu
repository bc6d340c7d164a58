// DMS-masked prefill attention on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory).
//
// Visible set of query i ([DMS-Qwen3], attention: the training score_mod's
// window and eviction gate at their hard inference limit):
//   V_i = { j <= i : i - j < w  or  alpha_j <= 0 }
// = band (i - w < j <= i)  U  kept prefix (j <= i - w, alpha_j <= 0).
//
// A CTA owns 128 query rows = NP = 128/g positions x the g query heads that
// share one KV head (row t = p * g + r), so every K/V tile feeds all g heads.
// Key tiles of 128 come from the contiguous band [i0 - w + 1, i1 - 1] and from
// the position-sorted kept list; evicted keys outside the window are never
// loaded.
//   S = Q K^T : tcgen05.mma M=128, N=128, K=16 x D/16, Q and K K-major in
//               128-byte-swizzled shared memory, S in TMEM columns [0, 128)
//   softmax   : 8 warps; row t is TMEM lane t, its 128 scores split between
//               two threads (columns 0-63 and 64-127).  The exponent reference
//               of a row is raised only when a tile's max exceeds it by 2^8, so
//               O is rescaled rarely (the final O / l is exact either way).
//   O += P V  : P (bf16, K-major) written to shared memory by the softmax
//               threads, V staged as MN-major B, O in TMEM columns [128, 128+D)
// Tiles arrive by TMA (no multicast): band keys/values straight from the input
// rows, kept ones from the position-sorted kept copy written by the
// compaction.  Two K/V stages and two S buffers let S(t+1) run on the tensor
// cores while the softmax of tile t runs; mbarriers order loads, S, and P V.
#include "dms_internal.cuh"

namespace dms {

#ifdef DMS_TRACE
__device__ unsigned long long g_dms_trace[2 * kTraceCtas * kTraceSlots];
#endif
// phases of tile 1 (tracing builds)
#define TC_MARK(tile, ph) \
  if ((tile) == 1) DMS_TRACE_MARK(0, (ph))

constexpr int kTcBN = 128;       // keys per tile
constexpr int kTcRows = 128;     // query rows per CTA (TMEM lanes)
constexpr int kTcThreads = 256;  // two threads per row

template <int D>
struct TcSmem {
  static constexpr int HALVES = D / 64;
  static constexpr int Q_BYTES = HALVES * kTcRows * 128;        // [half][128 rows][128 B]
  static constexpr int KV_BYTES = HALVES * kTcBN * 128;         // [half][128 keys][128 B]
  static constexpr int P_BYTES = (kTcBN / 64) * kTcRows * 128;  // [key half][128 rows][128 B]
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;       // 2 stages
  static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;  // 2 stages
  static constexpr int OFF_P = OFF_V + 2 * KV_BYTES;
  static constexpr int BYTES = OFF_P + P_BYTES;
  static constexpr uint32_t TMEM_COLS = 512;  // S double buffer: 2 x 128 columns, O: D columns at 256
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_attn_prefill_tc(CacheView c, int T, __nv_bfloat16* o, const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ CUtensorMap kkmap, const __grid_constant__ CUtensorMap kvmap) {
  using L = TcSmem<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sb = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = sb + L::OFF_Q;
  unsigned char* sP = sb + L::OFF_P;
  __shared__ __align__(16) int kpos[2][kTcBN];
  __shared__ float s_tmax[2][kTcRows];
  __shared__ float s_lpart[kTcRows];
  __shared__ float s_lsum[kTcRows];
  __shared__ uint32_t tmem_base;
  __shared__ __align__(8) uint64_t bar_q, bar_k[2], bar_v[2], bar_s[2], bar_pv;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (kTcRows - 1);  // TMEM lane / query row
  const int half = tid >> 7;            // which 64 key columns (and D/2 output columns)
  const int g = c.Hq / c.Hkv, NP = kTcRows / g;
  const int nqb = (T + NP - 1) / NP;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);  // heavy (late) blocks first
  const int h = blockIdx.y, b = blockIdx.z, w = c.w;
  const int i0 = qb * NP, i1 = min(T, i0 + NP);
  const int bh = b * c.Hkv + h;
  const int* kept = c.kept + static_cast<long>(bh) * c.max_pos;
  const int nk = (i1 - w > 0) ? c.kept_upto[static_cast<long>(bh) * (c.max_pos + 1) + (i1 - w)] : 0;
  const int jlo = max(0, i0 - w + 1), jhi = i1 - 1;
  const int n_kept_tiles = (nk + kTcBN - 1) / kTcBN;
  const int ntiles = n_kept_tiles + (jhi - jlo + kTcBN) / kTcBN;
  const int i_row = i0 + row / g, r_row = row % g;

  // position of key row `row` of a tile (-1: absent)
  auto key_pos = [&](int tile) -> int {
    if (tile < n_kept_tiles) {
      const int kidx = tile * kTcBN + row;
      return kidx < nk ? kept[kidx] : -1;
    }
    const int jj = jlo + (tile - n_kept_tiles) * kTcBN + row;
    return jj <= jhi ? jj : -1;
  };
  // TMA loads of a tile's keys or values into stage `st` (thread 0): band
  // tiles straight from the input rows, kept tiles from the kept copy
  auto load_kv = [&](int tile, int st, bool is_v) {
    unsigned char* dst = sb + (is_v ? L::OFF_V : L::OFF_K) + st * L::KV_BYTES;
    uint64_t* bar = is_v ? &bar_v[st] : &bar_k[st];
    mbar_expect_tx(bar, L::KV_BYTES);
    for (int hf = 0; hf < L::HALVES; ++hf) {
      if (tile < n_kept_tiles)
        tma_load_2d(dst + hf * (kTcBN * 128), is_v ? &kvmap : &kkmap, hf * 64, bh * c.max_pos + tile * kTcBN, bar);
      else
        tma_load_3d(dst + hf * (kTcBN * 128), is_v ? &vmap : &kmap, hf * 64, h,
                    b * T + jlo + (tile - n_kept_tiles) * kTcBN, bar);
    }
  };

  if (tid == 0) {
    mbar_init(&bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_k[i], 1);
      mbar_init(&bar_v[i], 1);
      mbar_init(&bar_s[i], 1);
    }
    mbar_init(&bar_pv, 1);
    fence_mbar_init();
    s_abort = 0;
    mbar_expect_tx(&bar_q, L::Q_BYTES);
    for (int hf = 0; hf < L::HALVES; ++hf) tma_load_3d(sQ + hf * (kTcRows * 128), &qmap, hf * 64, h * g, b * T + i0, &bar_q);
    load_kv(0, 0, false);
    load_kv(0, 0, true);
    if (ntiles > 1) {
      load_kv(1, 1, false);
      load_kv(1, 1, true);
    }
  }
  if (warp == 0) tmem_alloc(&tmem_base, L::TMEM_COLS);
  if (half == 0) kpos[0][row] = key_pos(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tmem_o = tmem + lane_off + 256 + half * (D / 2);  // this thread's D/2 output columns
  constexpr uint32_t IDESC_S = umma_idesc_bf16(128, kTcBN, 0);
  constexpr uint32_t IDESC_O = umma_idesc_bf16(128, D, 1);
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  float m_ref = -INFINITY, l_part = 0.f;

  // S(t) = Q K(t)^T into TMEM buffer t & 1 (thread 0)
  auto issue_s = [&](int tile) -> bool {
    const int st = tile & 1;
    if (!mbar_wait_bounded(&bar_k[st], (tile >> 1) & 1)) return false;
    tc_fence_after();
    const uint32_t qa = smem_u32(sQ), ka = smem_u32(sb + L::OFF_K + st * L::KV_BYTES);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t off = (ks / 4) * (kTcRows * 128) + (ks % 4) * 32;
      const uint32_t koff = (ks / 4) * (kTcBN * 128) + (ks % 4) * 32;
      umma_bf16(tmem + st * kTcBN, umma_desc_sw128(qa + off, 16, 1024), umma_desc_sw128(ka + koff, 16, 1024),
                IDESC_S, ks > 0 ? 1u : 0u);
    }
    umma_commit(&bar_s[st]);
    return true;
  };
  if (tid == 0) {
    if (!mbar_wait_bounded(&bar_q, 0) || !issue_s(0)) {
      set_status(c.ctrl, DMS_ST_TIMEOUT);
      s_abort = 1;
    }
  }

  for (int tile = 0; tile < ntiles; ++tile) {
    const int st = tile & 1;
    const bool kept_tile = tile < n_kept_tiles;
    const int j_next = tile + 1 < ntiles ? key_pos(tile + 1) : -1;  // read now, stored after the softmax
    TC_MARK(tile, 0);
    // next S on the tensor cores while this tile's softmax runs
    if (tid == 0 && !s_abort && tile + 1 < ntiles && !issue_s(tile + 1)) {
      set_status(c.ctrl, DMS_ST_TIMEOUT);
      s_abort = 1;
    }
    if (!mbar_wait_bounded(&bar_s[st], (tile >> 1) & 1)) {
      if (tid == 0) set_status(c.ctrl, DMS_ST_TIMEOUT);
      s_abort = 1;
    }
    tc_fence_after();
    TC_MARK(tile, 2);
    // K stage st is free (S(tile) complete): fetch the keys of tile + 2
    if (tid == 0 && tile + 2 < ntiles) load_kv(tile + 2, st, false);

    // ---- softmax: this thread's 64 scores of row `row` ----
    uint32_t sr[64];
    tmem_ld32_nowait(tmem + lane_off + st * kTcBN + half * 64, sr);
    tmem_ld32_nowait(tmem + lane_off + st * kTcBN + half * 64 + 32, sr + 32);
    tmem_wait_ld();
    TC_MARK(tile, 6);
    // visible: lo <= j <= hi (kept tile: 0 <= j <= i - w; band: i - w < j <= i); absent keys are -1
    const int lo = kept_tile ? 0 : max(0, i_row - w + 1);
    const int hi = kept_tile ? i_row - w : i_row;
    float x[64];
    float tmax = -INFINITY;
#pragma unroll
    for (int n4 = 0; n4 < 16; ++n4) {
      const int4 jv = reinterpret_cast<const int4*>(kpos[st] + half * 64)[n4];
      const int js[4] = {jv.x, jv.y, jv.z, jv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = n4 * 4 + e;
        x[n] = (js[e] >= lo && js[e] <= hi) ? __uint_as_float(sr[n]) * sl2 : -INFINITY;
        tmax = fmaxf(tmax, x[n]);
      }
    }
    s_tmax[half][row] = tmax;
    __syncthreads();
    if (s_abort) break;
    tmax = fmaxf(s_tmax[0][row], s_tmax[1][row]);
    TC_MARK(tile, 7);
    // raise the reference only when this tile exceeds it by more than 2^8
    const bool raise = tmax > m_ref + 8.0f;
    float factor = 1.0f;
    if (raise) {
      factor = (m_ref == -INFINITY) ? 0.0f : ex2_approx(m_ref - tmax);
      m_ref = tmax;
      l_part *= factor;
    }
    const float m_use = m_ref == -INFINITY ? 0.f : m_ref;  // a fully masked row so far: all p = 0
    uint32_t pk[32];
    float psum = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float p0 = ex2_approx(x[2 * e] - m_use);
      const float p1 = ex2_approx(x[2 * e + 1] - m_use);
      psum += p0 + p1;
      pk[e] = pack_bf16(p0, p1);
    }
    l_part += psum;
    // P(tile - 1) V has finished with the P buffer, with O and with V stage st ^ 1
    if (tile > 0 && !mbar_wait_bounded(&bar_pv, (tile - 1) & 1)) {
      if (tid == 0) set_status(c.ctrl, DMS_ST_TIMEOUT);
      s_abort = 1;
    }
    tc_fence_after();
    if (tid == 0 && tile >= 1 && tile + 1 < ntiles) load_kv(tile + 1, st ^ 1, true);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch)
      *reinterpret_cast<uint4*>(sP + half * (kTcRows * 128) + swz(row, ch)) =
          make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
    TC_MARK(tile, 8);
    // rescale this thread's half of O in tensor memory where the reference moved
    if (tile > 0 && __any_sync(0xffffffffu, raise && factor != 1.0f)) {
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        float ov[32];
        tmem_ld32(tmem_o + c0, ov);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) ov[jj] *= factor;
        tmem_st32(tmem_o + c0, ov);
      }
    }
    if (half == 0) kpos[st ^ 1][row] = j_next;  // the next tile's key positions
    TC_MARK(tile, 3);
    fence_proxy_async();  // P visible to the tensor cores
    tc_fence_before();
    __syncthreads();
    if (s_abort) break;
    if (tid == 0) {
      if (!mbar_wait_bounded(&bar_v[st], (tile >> 1) & 1)) {
        set_status(c.ctrl, DMS_ST_TIMEOUT);
        s_abort = 1;
      } else {
        tc_fence_after();
        const uint32_t pa = smem_u32(sP), va = smem_u32(sb + L::OFF_V + st * L::KV_BYTES);
#pragma unroll
        for (int ks = 0; ks < kTcBN / 16; ++ks) {
          const uint32_t poff = (ks / 4) * (kTcRows * 128) + (ks % 4) * 32;
          umma_bf16(tmem + 256, umma_desc_sw128(pa + poff, 16, 1024),
                    umma_desc_sw128(va + ks * 16 * 128, kTcBN * 128, 1024), IDESC_O, (tile > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&bar_pv);
      }
    }
    TC_MARK(tile, 4);
  }

  // wait for the last P V, then write O / l (l = the two halves' partial sums)
  if (half == 1) s_lpart[row] = l_part;
  __syncthreads();
  if (half == 0) s_lsum[row] = l_part + s_lpart[row];
  __syncthreads();
  if (!s_abort && ntiles > 0) {
    if (!mbar_wait_bounded(&bar_pv, (ntiles - 1) & 1) && tid == 0) set_status(c.ctrl, DMS_ST_TIMEOUT);
    tc_fence_after();
    const float inv = s_lsum[row] > 0.f ? 1.f / s_lsum[row] : 0.f;
    __nv_bfloat16* orow = o + ((static_cast<long>(b) * T + i_row) * c.Hq + h * g + r_row) * D + half * (D / 2);
#pragma unroll
    for (int c0 = 0; c0 < D / 2; c0 += 32) {
      float ov[32];
      tmem_ld32(tmem_o + c0, ov);
      if (i_row < T) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 pkk;
          pkk.x = pack_bf16(ov[e] * inv, ov[e + 1] * inv);
          pkk.y = pack_bf16(ov[e + 2] * inv, ov[e + 3] * inv);
          pkk.z = pack_bf16(ov[e + 4] * inv, ov[e + 5] * inv);
          pkk.w = pack_bf16(ov[e + 6] * inv, ov[e + 7] * inv);
          *reinterpret_cast<uint4*>(orow + c0 + e) = pkk;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

template <int D>
static cudaError_t launch_tc(const CacheView& c, int T, void* o, const PrefillMaps& m, cudaStream_t s) {
  const size_t smem = TcSmem<D>::BYTES + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_attn_prefill_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int g = c.Hq / c.Hkv, NP = kTcRows / g;
  dim3 grid((T + NP - 1) / NP, c.Hkv, c.B);
  k_attn_prefill_tc<D><<<grid, kTcThreads, smem, s>>>(c, T, static_cast<__nv_bfloat16*>(o), m.q, m.k, m.v, m.kept_k,
                                                      m.kept_v);
  return cudaGetLastError();
}

cudaError_t launch_prefill_attention_tc(const CacheView& c, int T, void* o, const PrefillMaps& maps, cudaStream_t s) {
  return c.D == 64 ? launch_tc<64>(c, T, o, maps, s) : launch_tc<128>(c, T, o, maps, s);
}

}  // namespace dms

#ifdef DMS_TRACE
extern "C" __attribute__((visibility("default"))) int dms_debug_trace_read_prefill(void* host, size_t bytes) {
  const size_t n = sizeof(dms::g_dms_trace) < bytes ? sizeof(dms::g_dms_trace) : bytes;
  return cudaMemcpyFromSymbol(host, dms::g_dms_trace, n) == cudaSuccess ? 0 : -3;
}
#endif
