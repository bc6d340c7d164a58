// Cache initialisation, decision logits and the neuron / rotary pre-pass.
#include "dms_internal.cuh"

namespace dms {

// ---------------------------------------------------------------------------
// Initialise (or reset) a cache: positions and counts to zero, preallocated
// pages granted row-major over (layer, batch, kv-head, page), page scales to
// zero, control words cleared, the page counter at the first free page.
// ---------------------------------------------------------------------------
__global__ void k_init(CacheView c) {
  const long nbh = static_cast<long>(c.L) * c.B * c.Hkv;
  const long npt = nbh * c.maxp;
  const long n = max(max(npt, static_cast<long>(c.pool_pages)), static_cast<long>(CTRL_WORDS));
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    if (i < npt) {
      const long lbh = i / c.maxp;
      const int p = static_cast<int>(i % c.maxp);
      c.page_table[i] = p < c.pre_pages ? static_cast<int>(lbh * c.pre_pages + p) : -1;
    }
    if (i < nbh) {
      c.npages[i] = c.pre_pages;
      c.count[i] = 0;
      c.plan[i] = make_int4(0, 0, 0, 0);
      c.plan[nbh + i] = make_int4(0, 0, 0, 0);
    }
    if (i < static_cast<long>(c.B) * c.Hkv) c.head_done[i] = 0;
    if (i < static_cast<long>(c.L) * c.B) c.pos[i] = 0;
    if (i < c.pool_pages) {
      c.k_scale[i] = 0.0f;
      c.v_scale[i] = 0.0f;
    }
    if (i < CTRL_WORDS) c.ctrl[i] = (i == CTRL_NEXT_PAGE) ? static_cast<int>(nbh * c.pre_pages) : 0;
  }
}

cudaError_t launch_init(const CacheView& c, bool full, cudaStream_t s) {
  if (full) {
    // Zero the page pools once: rows past a head's count are read (and masked)
    // by the attention tiles, so they must hold finite values.
    const size_t eb = c.kv_dtype == DMS_F32 ? 4 : c.kv_dtype == DMS_BF16 ? 2 : 1;
    const size_t pool_bytes = static_cast<size_t>(c.pool_pages) * c.P * c.D * eb;
    cudaError_t e = cudaMemsetAsync(c.k_pool, 0, pool_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(c.v_pool, 0, pool_bytes, s);
    // the kept copies too: tiles read (and mask) rows past the kept count
    const size_t kept_bytes = static_cast<size_t>(c.B) * c.Hkv * c.max_pos * c.D * 2;
    if (e == cudaSuccess && c.kept_k) e = cudaMemsetAsync(c.kept_k, 0, kept_bytes, s);
    if (e == cudaSuccess && c.kept_v) e = cudaMemsetAsync(c.kept_v, 0, kept_bytes, s);
    if (e != cudaSuccess) return e;
  }
  const long nbh = static_cast<long>(c.L) * c.B * c.Hkv;
  const long n = max(max(nbh * c.maxp, static_cast<long>(c.pool_pages)), static_cast<long>(CTRL_WORDS));
  const int grid = static_cast<int>(min((n + 255) / 256, 4096L));
  k_init<<<grid, 256, 0, s>>>(c);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Decision logits from the adapter: alpha = (W_h . RMSNorm_gamma(x) + bias_h)
// * scale - offset.  RMSNorm's gamma is folded into W in shared memory, and the
// 1/rms factor is applied after the dot product:
//   W_h . (x * inv * gamma) = inv * ((W_h * gamma) . x).
// Each warp handles kTok tokens at once so each W element read from shared
// memory serves kTok tokens.  Supports Hkv <= 8.
// ---------------------------------------------------------------------------
constexpr int kTok = 4;

template <typename TA>
__global__ void __launch_bounds__(256) k_decide_proj(CacheView c, int T, DecideArgs a, float* alpha) {
  extern __shared__ float wg[];  // [Hkv][hidden]
  const int H = c.Hkv, hid = c.hidden;
  const TA* W = static_cast<const TA*>(a.W);
  const TA* gamma = static_cast<const TA*>(a.gamma);
  const TA* hs = static_cast<const TA*>(a.hidden);
  const TA* bias = static_cast<const TA*>(a.bias);
  for (int i = threadIdx.x; i < H * hid; i += blockDim.x) wg[i] = to_f(W[i]) * to_f(gamma[i % hid]);
  __syncthreads();

  constexpr int V = 16 / sizeof(TA);
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long gw = static_cast<long>(blockIdx.x) * warps + (threadIdx.x >> 5);
  const long nwarps = static_cast<long>(gridDim.x) * warps;
  const long ntok = static_cast<long>(c.B) * T;
  const int nvec = hid / V;
  const bool layer_mode = c.alpha_per == DMS_ALPHA_PER_LAYER;

  for (long tok0 = gw * kTok; tok0 < ntok; tok0 += nwarps * kTok) {
    float ss[kTok];
    float dot[kTok][8];
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
      ss[u] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) dot[u][j] = 0.f;
    }
    for (int vi = lane; vi < nvec; vi += 32) {
      float x[kTok][V];
#pragma unroll
      for (int u = 0; u < kTok; ++u) {
        const long tok = tok0 + u;
        if (tok < ntok) {
          uint4 raw = reinterpret_cast<const uint4*>(hs + tok * hid)[vi];
          unpack16(raw, x[u], static_cast<const TA*>(nullptr));
        } else {
#pragma unroll
          for (int e = 0; e < V; ++e) x[u][e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < V; ++e) ss[u] = fmaf(x[u][e], x[u][e], ss[u]);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < H) {
          const float* wp = wg + j * hid + vi * V;
#pragma unroll
          for (int e = 0; e < V; ++e) {
            const float wv = wp[e];
#pragma unroll
            for (int u = 0; u < kTok; ++u) dot[u][j] = fmaf(wv, x[u][e], dot[u][j]);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot[u][j] += __shfl_xor_sync(0xffffffffu, dot[u][j], o);
    }
    if (lane < kTok) {
      // lane u writes token tok0 + u (register arrays indexed with a constant)
#pragma unroll
      for (int u = 0; u < kTok; ++u) {
        if (u != lane) continue;
        const long tok = tok0 + u;
        if (tok >= ntok) continue;
        const int b = static_cast<int>(tok / T), t = static_cast<int>(tok % T);
        const float inv = 1.0f / sqrtf(ss[u] / static_cast<float>(hid) + c.rms_eps);
        float a0 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j >= H) continue;
          const int src = layer_mode ? 0 : j;
          float z = dot[u][src] * inv + (bias ? to_f(bias[src]) : 0.f);
          float al = z * c.alpha_scale - a.offset[b * a.offset_bstride + src];
          if (j == 0) a0 = al;
          alpha[(static_cast<long>(b) * H + j) * T + t] = layer_mode ? a0 : al;
        }
      }
    }
  }
}

// Decode-shaped variant (one token per sequence): one CTA per (kv-head, b),
// the hidden row and W_h read straight from global memory as 16-byte vectors.
template <typename TA>
__global__ void __launch_bounds__(256) k_decide_proj_row(CacheView c, DecideArgs a, float* alpha) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int src = c.alpha_per == DMS_ALPHA_PER_LAYER ? 0 : h;
  const int hid = c.hidden;
  constexpr int V = 16 / sizeof(TA);
  const uint4* x = reinterpret_cast<const uint4*>(static_cast<const TA*>(a.hidden) + static_cast<long>(b) * hid);
  const uint4* W = reinterpret_cast<const uint4*>(static_cast<const TA*>(a.W) + static_cast<long>(src) * hid);
  const uint4* gamma = reinterpret_cast<const uint4*>(a.gamma);
  float ss = 0.f, dot = 0.f;
  for (int vi = threadIdx.x; vi < hid / V; vi += blockDim.x) {
    float xv[V], wv[V], gv[V];
    unpack16(x[vi], xv, static_cast<const TA*>(nullptr));
    unpack16(W[vi], wv, static_cast<const TA*>(nullptr));
    unpack16(gamma[vi], gv, static_cast<const TA*>(nullptr));
#pragma unroll
    for (int e = 0; e < V; ++e) {
      ss = fmaf(xv[e], xv[e], ss);
      dot = fmaf(wv[e] * gv[e], xv[e], dot);
    }
  }
  __shared__ float red[2][32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) {
    red[0][wid] = ss;
    red[1][wid] = dot;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s2 = 0.f, d2 = 0.f;
    for (int i = 0; i < (blockDim.x >> 5); ++i) {
      s2 += red[0][i];
      d2 += red[1][i];
    }
    const TA* bias = static_cast<const TA*>(a.bias);
    const float inv = 1.0f / sqrtf(s2 / static_cast<float>(hid) + c.rms_eps);
    const float z = d2 * inv + (bias ? to_f(bias[src]) : 0.f);
    alpha[b * c.Hkv + h] = z * c.alpha_scale - a.offset[b * a.offset_bstride + src];
  }
}

cudaError_t launch_decide_proj(const CacheView& c, int T, const DecideArgs& a, float* alpha, cudaStream_t s) {
  if (T == 1) {
    dim3 grid(c.Hkv, c.B);
    if (c.act_dtype == DMS_BF16)
      k_decide_proj_row<__nv_bfloat16><<<grid, 256, 0, s>>>(c, a, alpha);
    else
      k_decide_proj_row<float><<<grid, 256, 0, s>>>(c, a, alpha);
    return cudaGetLastError();
  }
  const size_t smem = static_cast<size_t>(c.Hkv) * c.hidden * sizeof(float);
  const long ntok = static_cast<long>(c.B) * T;
  const long want = (ntok + 8 * kTok - 1) / (8 * kTok);
  const int grid = static_cast<int>(min(want, static_cast<long>(c.num_sms)));
  cudaError_t e;
  if (c.act_dtype == DMS_BF16) {
    e = cudaFuncSetAttribute(k_decide_proj<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_decide_proj<__nv_bfloat16><<<grid, 256, smem, s>>>(c, T, a, alpha);
  } else {
    e = cudaFuncSetAttribute(k_decide_proj<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_decide_proj<float><<<grid, 256, smem, s>>>(c, T, a, alpha);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Neuron decisions and rotary embedding, one thread per (token, row, i <
// D/2) element pair, in place:
//  1. (neuron source) alpha = x[D-1] * scale - offset for the key of head h or
//     the query of head h*g, read by the thread of pair i = D/2 - 1 of that
//     row; layer granularity takes head 0's value; then the decision element
//     of every head is set to zero;
//  2. (tables given) half-split rotation of every query and key row of the
//     token at position t (prefill), or at the sequence's current position
//     pos_dev[b] (decode, T == 1).
// ---------------------------------------------------------------------------
template <typename TA>
__global__ void k_neuron_rope(CacheView c, int T, const int* pos_dev, TA* q, TA* k, const float* offset, int ostride,
                              int do_alpha, float* alpha, const float* cos_t, const float* sin_t) {
  const int D = c.D, half = D / 2, g = c.Hq / c.Hkv;
  const bool key = c.alpha_source == DMS_ALPHA_KEY_NEURON;
  // with rotary tables every (token, row, i < D/2) pair, else only the
  // decision neuron of each head (its pair i = D/2 - 1)
  const int nrow = cos_t ? c.Hq + c.Hkv : c.Hkv;
  const int npair = cos_t ? half : 1;
  const long total = static_cast<long>(c.B) * T * nrow * npair;
  for (long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int i = cos_t ? static_cast<int>(idx % half) : half - 1;
    const long rt = idx / npair;
    int r = static_cast<int>(rt % nrow);
    const long tok = rt / nrow;
    if (!cos_t) r = key ? c.Hq + r : r * g;  // the neuron rows only
    const int b = static_cast<int>(tok / T), t = static_cast<int>(tok % T);
    TA* row = r < c.Hq ? q + (tok * c.Hq + r) * D : k + (tok * c.Hkv + (r - c.Hq)) * D;
    float x0 = to_f(row[i]), x1 = to_f(row[i + half]);
    // the decision neuron (the last element of each key, or of the first query
    // head of each group) is read, then zeroed, before the rotation
    const bool neuron_row = key ? r >= c.Hq : (r < c.Hq && r % g == 0);
    if (do_alpha && neuron_row && i == half - 1) {
      const int h = key ? r - c.Hq : r / g;
      if (c.alpha_per == DMS_ALPHA_PER_LAYER) {
        if (h == 0) {
          const float a = fmaf(x1, c.alpha_scale, -offset[b * ostride]);
          for (int hh = 0; hh < c.Hkv; ++hh) alpha[(static_cast<long>(b) * c.Hkv + hh) * T + t] = a;
        }
      } else {
        alpha[(static_cast<long>(b) * c.Hkv + h) * T + t] = fmaf(x1, c.alpha_scale, -offset[b * ostride + h]);
      }
      x1 = 0.f;
    }
    if (cos_t) {
      const int p = pos_dev ? pos_dev[b] + t : t;
      const float cv = cos_t[static_cast<long>(p) * half + i], sv = sin_t[static_cast<long>(p) * half + i];
      // each product and sum rounded separately (no fused multiply-add), so
      // the stored value does not depend on contraction choices
      row[i] = from_f<TA>(__fsub_rn(__fmul_rn(x0, cv), __fmul_rn(x1, sv)));
      row[i + half] = from_f<TA>(__fadd_rn(__fmul_rn(x1, cv), __fmul_rn(x0, sv)));
    } else {
      row[i + half] = from_f<TA>(x1);
    }
  }
}

cudaError_t launch_neuron_rope(const CacheView& c, int T, const int* pos_dev, void* q, void* k, const float* offset,
                               int offset_bstride, bool do_alpha, float* alpha, const float* cos_t,
                               const float* sin_t, cudaStream_t s) {
  const long total = static_cast<long>(c.B) * T * (cos_t ? (c.Hq + c.Hkv) * (c.D / 2) : c.Hkv);
  const int grid = static_cast<int>(max(1L, min((total + 255) / 256, static_cast<long>(c.num_sms) * 16)));
  if (c.act_dtype == DMS_BF16)
    k_neuron_rope<__nv_bfloat16><<<grid, 256, 0, s>>>(c, T, pos_dev, static_cast<__nv_bfloat16*>(q),
                                                       static_cast<__nv_bfloat16*>(k), offset, offset_bstride,
                                                       do_alpha ? 1 : 0, alpha, cos_t, sin_t);
  else
    k_neuron_rope<float><<<grid, 256, 0, s>>>(c, T, pos_dev, static_cast<float*>(q), static_cast<float*>(k), offset,
                                              offset_bstride, do_alpha ? 1 : 0, alpha, cos_t, sin_t);
  return cudaGetLastError();
}

}  // namespace dms
