// DMS-masked prefill attention.
//
// Query i sees key j iff j <= i and (i - j < w or alpha_j <= 0)
// ([DMS-Qwen3], attention: the training score_mod's sliding window and eviction
// gate at their hard inference limit).  The visible set splits into two
// disjoint parts that are each cheap to enumerate:
//   band:        i - w < j <= i                  (contiguous keys)
//   kept prefix: j <= i - w and alpha_j <= 0     (the position-sorted kept list)
// so a block of queries [i0, i1) reads the contiguous band
// [i0 - w + 1, i1 - 1] and the kept-list entries with position <= i1 - 1 - w,
// and never touches the evicted keys outside the window.
#include "dms_internal.cuh"

namespace dms {

// ---------------------------------------------------------------------------
// fp32 path (CUDA cores, exact fp32 arithmetic): one warp per query row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_attn_prefill_f32(CacheView c, int T, const float* q, const float* k,
                                                         const float* v, float* o) {
  const int lane = threadIdx.x & 31;
  const long row = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long nrows = static_cast<long>(c.B) * T * c.Hq;
  if (row >= nrows) return;
  const int hq = static_cast<int>(row % c.Hq);
  const long bt = row / c.Hq;
  const int b = static_cast<int>(bt / T), i = static_cast<int>(bt % T);
  const int g = c.Hq / c.Hkv, h = hq / g, D = c.D, w = c.w;
  const int per = D / 32;  // 2 or 4
  float qv[4], acc[4];
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  for (int e = 0; e < per; ++e) {
    qv[e] = q[row * D + lane * per + e] * scale;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int bh = b * c.Hkv + h;
  const int* kept = c.kept + static_cast<long>(bh) * c.max_pos;
  const int nk = i - w + 1 > 0 ? c.kept_upto[static_cast<long>(bh) * (c.max_pos + 1) + (i - w + 1)] : 0;
  const int jlo = max(0, i - w + 1);
  const int total = nk + (i - jlo + 1);
  for (int n = 0; n < total; ++n) {
    const int j = n < nk ? kept[n] : jlo + (n - nk);
    const float* kr = k + ((static_cast<long>(b) * T + j) * c.Hkv + h) * D + lane * per;
    float s = 0.f;
    for (int e = 0; e < per; ++e) s = fmaf(qv[e], kr[e], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float mn = fmaxf(m, s);
    const float corr = expf(m - mn);
    const float p = expf(s - mn);
    l = l * corr + p;
    const float* vr = v + ((static_cast<long>(b) * T + j) * c.Hkv + h) * D + lane * per;
    for (int e = 0; e < per; ++e) acc[e] = acc[e] * corr + p * vr[e];
    m = mn;
  }
  for (int e = 0; e < per; ++e) o[row * D + lane * per + e] = acc[e] / l;
}

// ---------------------------------------------------------------------------
// bf16 path: flash-attention tiles on mma.sync (m16n8k16, fp32 accumulators).
// CTA = 4 warps x 16 query rows of one (b, hq); key tiles of 64 rows are
// staged in shared memory with cp.async, double buffered.
// ---------------------------------------------------------------------------
constexpr int kBM = 64;
constexpr int kBN = 64;

template <int D>
struct PrefillSmem {
  static constexpr int LD = D + 8;  // padded row (elements): conflict-free ldmatrix
  __nv_bfloat16 q[kBM * LD];
  __nv_bfloat16 k[2][kBN * LD];
  __nv_bfloat16 v[2][kBN * LD];
  int kpos[2][kBN];
};

template <int D>
__global__ void __launch_bounds__(128) k_attn_prefill_bf16(CacheView c, int T, const __nv_bfloat16* q,
                                                          const __nv_bfloat16* k, const __nv_bfloat16* v,
                                                          __nv_bfloat16* o) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  PrefillSmem<D>& sm = *reinterpret_cast<PrefillSmem<D>*>(smem_raw);
  constexpr int LD = PrefillSmem<D>::LD;
  constexpr int KS = D / 16;  // k-steps over the head dimension
  constexpr int NT = D / 8;   // n-tiles of the output
  const int nqb = (T + kBM - 1) / kBM;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);  // heavy (late) blocks first
  const int hq = blockIdx.y, b = blockIdx.z;
  const int g = c.Hq / c.Hkv, h = hq / g, w = c.w;
  const int i0 = qb * kBM, i1 = min(T, i0 + kBM);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long kv_row_stride = static_cast<long>(c.Hkv) * D;
  const __nv_bfloat16* kbase = k + static_cast<long>(b) * T * kv_row_stride + static_cast<long>(h) * D;
  const __nv_bfloat16* vbase = v + static_cast<long>(b) * T * kv_row_stride + static_cast<long>(h) * D;
  const int bh = b * c.Hkv + h;
  const int* kept = c.kept + static_cast<long>(bh) * c.max_pos;
  const int nk = (i1 - w > 0) ? c.kept_upto[static_cast<long>(bh) * (c.max_pos + 1) + (i1 - w)] : 0;
  const int jlo = max(0, i0 - w + 1), jhi = i1 - 1;
  const int n_kept_tiles = (nk + kBN - 1) / kBN;
  const int n_band_tiles = (jhi - jlo + 1 + kBN - 1) / kBN;
  const int ntiles = n_kept_tiles + n_band_tiles;

  // Q tile
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  for (int idx = tid; idx < kBM * CPR; idx += 128) {
    const int r = idx / CPR, ch = idx % CPR;
    const int i = i0 + r;
    const __nv_bfloat16* src = q + ((static_cast<long>(b) * T + min(i, T - 1)) * c.Hq + hq) * D + ch * 8;
    cp_async16_zfill(&sm.q[r * LD + ch * 8], src, i < T);
  }
  cp_async_commit();

  // Two threads per key row: the row's position is read once, then each thread
  // issues its half of the row's 16-byte copies.
  auto load_tile = [&](int tile, int buf) {
    const int n = tid >> 1, part = tid & 1;
    int j;
    if (tile < n_kept_tiles) {
      const int kidx = tile * kBN + n;
      j = kidx < nk ? kept[kidx] : -1;
    } else {
      const int jj = jlo + (tile - n_kept_tiles) * kBN + n;
      j = jj <= jhi ? jj : -1;
    }
    if (part == 0) sm.kpos[buf][n] = j;
    const long off = static_cast<long>(max(j, 0)) * kv_row_stride;
#pragma unroll
    for (int cc = 0; cc < CPR / 2; ++cc) {
      const int ch = part * (CPR / 2) + cc;
      cp_async16_zfill(&sm.k[buf][n * LD + ch * 8], kbase + off + ch * 8, j >= 0);
      cp_async16_zfill(&sm.v[buf][n * LD + ch * 8], vbase + off + ch * 8, j >= 0);
    }
    cp_async_commit();
  };

  if (ntiles > 0) load_tile(0, 0);
  cp_async_wait<1>();
  __syncthreads();

  // Q fragments (A operand, rows warp*16 .. +15)
  uint32_t qa[KS][4];
  {
    const int mi = lane >> 3, rr = lane & 7;
    const int row = warp * 16 + (mi & 1) * 8 + rr;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int col = ks * 16 + (mi >> 1) * 8;
      ldmatrix_x4(qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], smem_u32(&sm.q[row * LD + col]));
    }
  }

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));  // log2(e)/sqrt(D)
  const int ia = i0 + warp * 16 + (lane >> 2), ib = ia + 8;

  for (int tile = 0; tile < ntiles; ++tile) {
    const int buf = tile & 1;
    if (tile + 1 < ntiles) load_tile(tile + 1, buf ^ 1);
    else cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const bool kept_tile = tile < n_kept_tiles;
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    {
      const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          const int n = np * 16 + (mi >> 1) * 8 + rr;
          const int col = ks * 16 + (mi & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(b0, b1, b2, b3, smem_u32(&sm.k[buf][n * LD + col]));
          uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
          mma_bf16_16816(s[2 * np], qa[ks], bb0);
          mma_bf16_16816(s[2 * np + 1], qa[ks], bb1);
        }
      }
    }
    // mask + online softmax (rows ia, ib)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = nt * 8 + 2 * (lane & 3) + (e & 1);
        const int i = e < 2 ? ia : ib;
        const int j = sm.kpos[buf][n];
        bool vis;
        if (kept_tile)
          vis = j >= 0 && j <= i - w;
        else
          vis = j >= 0 && j <= i && i - j < w;
        const float x = vis ? s[nt][e] * sl2 : -INFINITY;
        s[nt][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float corr[2], mu[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float mn = fmaxf(mrow[r], mx[r]);
      mu[r] = mn == -INFINITY ? 0.f : mn;
      corr[r] = exp2f(mrow[r] - mu[r]);
      mrow[r] = mn;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[nt][e] - mu[e >> 1]);
        s[nt][e] = p;
        rs[e >> 1] += p;
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) lrow[r] = lrow[r] * corr[r] + rs[r];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      acc[nt][0] *= corr[0];
      acc[nt][1] *= corr[0];
      acc[nt][2] *= corr[1];
      acc[nt][3] *= corr[1];
    }
    // O += P V
    {
      const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int dp = 0; dp < NT / 2; ++dp) {
          const int n = kk * 16 + (mi & 1) * 8 + rr;
          const int col = dp * 16 + (mi >> 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(&sm.v[buf][n * LD + col]));
          uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
          mma_bf16_16816(acc[2 * dp], pa, bb0);
          mma_bf16_16816(acc[2 * dp + 1], pa, bb1);
        }
      }
    }
    __syncthreads();
  }
  // row sums across the quad, normalise, store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  const float inv0 = lrow[0] > 0.f ? 1.f / lrow[0] : 0.f;
  const float inv1 = lrow[1] > 0.f ? 1.f / lrow[1] : 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int col = nt * 8 + 2 * (lane & 3);
    if (ia < T)
      *reinterpret_cast<uint32_t*>(o + ((static_cast<long>(b) * T + ia) * c.Hq + hq) * D + col) =
          pack_bf16(acc[nt][0] * inv0, acc[nt][1] * inv0);
    if (ib < T)
      *reinterpret_cast<uint32_t*>(o + ((static_cast<long>(b) * T + ib) * c.Hq + hq) * D + col) =
          pack_bf16(acc[nt][2] * inv1, acc[nt][3] * inv1);
  }
}

template <int D>
static cudaError_t launch_bf16(const CacheView& c, int T, const void* q, const void* k, const void* v, void* o,
                               cudaStream_t s) {
  const size_t smem = sizeof(PrefillSmem<D>);
  cudaError_t e = cudaFuncSetAttribute(k_attn_prefill_bf16<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((T + kBM - 1) / kBM, c.Hq, c.B);
  k_attn_prefill_bf16<D><<<grid, 128, smem, s>>>(c, T, static_cast<const __nv_bfloat16*>(q),
                                                 static_cast<const __nv_bfloat16*>(k),
                                                 static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(o));
  return cudaGetLastError();
}

cudaError_t launch_prefill_attention(const CacheView& c, int T0, int T, const void* q, const void* k, const void* v,
                                     void* o, const PrefillMaps* maps, cudaStream_t s) {
  // a later chunk of a chunked prefill reads the window and kept copies: the
  // tcgen05 kernel only (the host refuses other shapes for such calls)
  if (T0 > 0) return maps && maps->valid ? launch_prefill_attention_tc(c, T0, T, o, *maps, s) : cudaErrorNotSupported;
  if (c.act_dtype == DMS_F32) {
    const long nrows = static_cast<long>(c.B) * T * c.Hq;
    const int grid = static_cast<int>((nrows * 32 + 255) / 256);
    k_attn_prefill_f32<<<grid, 256, 0, s>>>(c, T, static_cast<const float*>(q), static_cast<const float*>(k),
                                            static_cast<const float*>(v), static_cast<float*>(o));
    return cudaGetLastError();
  }
  // bf16: the tcgen05 kernel; shapes it does not cover (g not a power of two
  // up to 16, or inputs not 16-byte aligned for TMA) take the mma.sync kernel
  if (maps && maps->valid) return launch_prefill_attention_tc(c, 0, T, o, *maps, s);
  return c.D == 64 ? launch_bf16<64>(c, T, q, k, v, o, s) : launch_bf16<128>(c, T, q, k, v, o, s);
}

}  // namespace dms
