// Internal definitions shared by the CUDA translation units of libdms.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dms.h"

namespace dms {

// ---------------------------------------------------------------------------
// Control words at the start of the cache buffer.
// ---------------------------------------------------------------------------
enum Ctrl {
  CTRL_STATUS = 0,       // sticky DMS_ST_* bits
  CTRL_NEXT_PAGE = 1,    // next page id the ascending counter hands out
  CTRL_DONE_SCAN = 2,    // arrival counter of the prefill scan CTAs
  CTRL_STEP64 = 4,       // (64-bit, words 4-5) fused decode step: CTAs arrived, pages granted
  CTRL_WORDS = 64
};

// Device view of one cache: sizes and device pointers into the caller buffer.
struct CacheView {
  int L, B, Hq, Hkv, D, hidden, w, P, maxp, cap, pool_pages, pre_pages, max_pos;
  int kv_dtype, act_dtype, alpha_per, alpha_source, disable, decode_kernel, shift;
  float alpha_scale, rms_eps;
  int num_sms;
  int* ctrl;
  int* pos;         // [L,B]
  int* count;       // [L,B,Hkv]
  int* npages;      // [L,B,Hkv]
  int* page_table;  // [L,B,Hkv,maxp]
  int* slot_pos;    // [L,B,Hkv,cap]
  int* ring;        // [L,B,Hkv,w]
  int* carry;       // [L,B,Hkv] decision shift +1: the newest token's own decision
  int4* plan;       // [2][L,B,Hkv] plan of the next append, by parity of its position (next_plan)
  int* kept;        // [B,Hkv,max_pos]   prefill scratch: kept positions, ascending
  int* kept_count;  // [B,Hkv]
  int* kept_upto;   // [B,Hkv,max_pos+1] prefill scratch: kept tokens before position t
  int* scan;        // [B,Hkv][scan_stride] prefill scratch of the two scan launches
  int scan_stride;
  void* kept_k;     // [B*Hkv, max_pos, D] prefill scratch (bf16 activations): kept keys in list order
  void* kept_v;     //                      and values
  void* win_k;      // [B*Hkv, w, D] prefill scratch (bf16 activations): the keys of the last w positions
  void* win_v;      //                before a later chunk of a chunked prefill, and the values
  int* head_done;   // [B*Hkv] arrival counters of the attention CTAs (self-resetting)
  float* part_acc;  // [items_cap, g, D]   decode split-K partials, indexed by work item
  float* part_ml;   // [items_cap, g, 2]  (running max, running sum)
  int items_cap;
  float* k_scale;   // [pool_pages]
  float* v_scale;
  void* k_pool;     // [pool_pages, P, D]
  void* v_pool;
};

constexpr unsigned RING_EVICT = 0x80000000u;
constexpr int RING_SLOT_MASK = 0x7FFFFFFF;

// The eviction mark stored with token t, appended with its own decision `dec`
// (logit > 0, eviction enabled), under the cache's decision shift: 0, its own
// decision; +1, the previous token's (carried per head); -1, unmarked until the
// next token, and `dec` marks token t - 1 in its ring entry now.  Called by the
// one thread that appends to head li.
__device__ __forceinline__ bool shifted_mark(const CacheView& c, long li, int t, bool dec) {
  if (c.shift == 1) {
    const bool m = c.carry[li] != 0;
    c.carry[li] = dec ? 1 : 0;
    return m;
  }
  if (c.shift == -1) {
    if (t >= 1 && dec) {
      int* e = c.ring + li * c.w + (t - 1) % c.w;
      *e = *e | static_cast<int>(RING_EVICT);
    }
    return false;
  }
  return dec;
}

// Bounded spin limit for every device-side wait.
constexpr long long kSpinLimit = 1ll << 26;

__device__ __forceinline__ void set_status(int* ctrl, int bits) { atomicOr(&ctrl[CTRL_STATUS], bits); }

// Plan entry of head li for the append of the token at position t (the plan is
// double-buffered by the parity of t so one decode step can read its own plan
// while writing the next one).  It also snapshots the head's retained count
// and page count before that append: a decode launch that appends reads every
// head's count from here, never from the live count its own CTAs update.
__device__ __forceinline__ int4* plan_at(const CacheView& c, long li, int t) {
  return c.plan + static_cast<long>(t & 1) * c.L * c.B * c.Hkv + li;
}

// ---------------------------------------------------------------------------
// Element helpers
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Rotary embedding of one pair (x_i, x_{i+D/2}) by the table entries (c, s), in
// fp64.  Each product of a bf16 or fp32 element with an fp32 table entry has at
// most 48 significant bits and is exact in fp64, so each output is the exact
// rotation rounded once.
__device__ __forceinline__ void rotate64(double a, double b, double c, double s, double& y0, double& y1) {
  y0 = __dsub_rn(__dmul_rn(a, c), __dmul_rn(b, s));
  y1 = __dadd_rn(__dmul_rn(b, c), __dmul_rn(a, s));
}

// fp64 -> bf16 with one round-to-nearest-even step: the value is first
// narrowed to fp32 rounding to odd (truncate, then set the last bit when
// anything was dropped), which keeps 16 more bits than bf16 carries, so the
// final fp32 -> bf16 rounding decides exactly as a direct rounding would.
__device__ __forceinline__ float f64_to_f32_odd(double x) {
  float r = __double2float_rz(x);
  if (static_cast<double>(r) != x) r = __int_as_float(__float_as_int(r) | 1);
  return r;
}
template <typename T>
__device__ __forceinline__ T from_f64(double x);
template <>
__device__ __forceinline__ float from_f64<float>(double x) { return __double2float_rn(x); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f64<__nv_bfloat16>(double x) {
  return __float2bfloat16_rn(f64_to_f32_odd(x));
}

// 16 bytes of the RMSNorm weight gamma (vector vi), or of ones when there is
// none (the score source has no normalisation).
template <typename TA>
__device__ __forceinline__ uint4 gamma16(const void* g, long vi) {
  if (g) return reinterpret_cast<const uint4*>(g)[vi];
  const unsigned one = sizeof(TA) == 2 ? 0x3F803F80u : 0x3F800000u;
  return make_uint4(one, one, one, one);
}

// Decision logit of the adapter sources from dot = W_h . (x * gamma), the
// sum of squares ss of the hidden row x (hid elements), the bias and the
// offset: PROJ, alpha = (dot / rms(x) + bias) * alpha_scale - offset with
// rms(x) = sqrt(ss / hid + rms_eps); SCORE_LINEAR (a KVzap-style importance
// score, gamma absent), alpha = offset - (dot + bias) with the offset as the
// pruning threshold: a token scoring below it is marked.
__device__ __forceinline__ float adapter_logit(const CacheView& c, float dot, float ss, int hid, float bias,
                                               float offset) {
  if (c.alpha_source == DMS_ALPHA_SCORE_LINEAR) return offset - (dot + bias);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(hid) + c.rms_eps);
  return (dot * inv + bias) * c.alpha_scale - offset;
}

// Unpack a 16-byte vector into floats (8 bf16 or 4 fp32).
template <typename T>
struct Vec16 {
  static constexpr int N = 16 / sizeof(T);
};

__device__ __forceinline__ void unpack16(const uint4& u, float* f, const __nv_bfloat16*) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void unpack16(const uint4& u, float* f, const float*) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}

// FP8 E4M3 encode with round-to-nearest-even and saturation to +-448.
__device__ __forceinline__ uint8_t fp8_encode(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ float fp8_decode(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(h));
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024,
// a multiple of 32).  `tmp` holds 32 ints of shared memory.  Returns the
// exclusive prefix; *total receives the block sum.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = lane < nw ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    tmp[lane] = s;  // inclusive prefix of warp sums
  }
  __syncthreads();
  int warp_base = wid ? tmp[wid - 1] : 0;
  *total = tmp[nw - 1];
  __syncthreads();
  return warp_base + x - v;
}

// ---------------------------------------------------------------------------
// PTX wrappers: cp.async, ldmatrix, mma.sync, mbarrier, TMA tile loads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool valid) {
  int src_bytes = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Two fp64 values rounded once each (see f64_to_f32_odd) into a bf16 pair.
__device__ __forceinline__ uint32_t pack_bf16_f64(double lo, double hi) {
  return pack_bf16(f64_to_f32_odd(lo), f64_to_f32_odd(hi));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait that parks the warp: each try may suspend the thread for up to
// 20 us until the phase completes, so waiting warps leave their issue slots to
// the others; gives up (returns false) after about 2.6 s.
__device__ __forceinline__ bool mbar_wait_parked(uint64_t* bar, uint32_t parity) {
  for (int i = 0; i < (1 << 17); ++i) {
    uint32_t ok;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    if (ok) return true;
  }
  return false;
}
// Bounded wait: returns false (and the caller must give up) after `tries`
// tries (kSpinLimit unless a caller asks for fewer).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, long long tries = kSpinLimit) {
  for (long long i = 0; i < tries; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// 2-D TMA tile load (no multicast) into shared memory, completing on `bar`.
// warm a tile of a 2D tensor map into L2 (no shared memory, no completion)
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];\n" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];\n" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in tensor memory).
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor: start address, leading / stride byte
// offsets (16-byte units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}
// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator,
// K-major A, B K-major (b_mn_major = 0) or MN-major (1), M x N tile.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn_major) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc));
}
// The same product with A (M x K, K-major) read from tensor memory: row m in
// lane m, 16-bit elements packed two per 32-bit column from column tmem_a on.
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                             uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(dst_smem)),
               "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
// 32 consecutive fp32 columns of this thread's TMEM lane (warp w owns lanes 32w..32w+31).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}
// 32 consecutive 32-bit columns of this thread's lane from raw words, without
// waiting (tcgen05.wait::st orders them before a release).
__device__ __forceinline__ void tmem_st32_nowait(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// ---------------------------------------------------------------------------
// Host-side launchers (one per translation unit).
// ---------------------------------------------------------------------------
struct DecideArgs {
  const void* hidden;
  const void* gamma;
  const void* W;
  const void* bias;
  const float* offset;
  int offset_bstride;
  // a decode launch over several layers: elements from one layer's gamma, W,
  // bias and offsets to the next (hidden rows continue layer by layer)
  long gamma_lstride, w_lstride, bias_lstride, offset_lstride;
};

cudaError_t launch_init(const CacheView& c, bool full, cudaStream_t s);
// hmap: tensor map of the hidden rows [B*T, hidden] (bf16, 128-byte swizzle,
// box 64 x 64), or null (CUDA-core kernel).
cudaError_t launch_decide_proj(const CacheView& c, int T, const DecideArgs& a, float* alpha, const CUtensorMap* hmap,
                               cudaStream_t s);
// pdl: launched as a programmatic dependent of the previous kernel on the
// stream (the kernels wait for it before reading, then let the next kernel
// start its prologue).
cudaError_t launch_neuron_rope(const CacheView& c, int T, const int* pos_dev, void* q, void* k, const float* offset,
                               int offset_bstride, bool do_alpha, float* alpha, const float* cos_t,
                               const float* sin_t, cudaStream_t s, bool pdl = false);
// Prefill of T tokens at positions T0 .. T0 + T - 1 (T0 > 0: a later chunk of
// a chunked prefill; launch_prefill_context rebuilds the kept list, kept copy
// and window copy of the layer first).
size_t prefill_scan_smem(const CacheView& c, int T0, int T);
// ints of scan scratch per (b, h)
int prefill_scan_stride(int max_pos, int w);
cudaError_t launch_prefill_context(const CacheView& c, int layer, int T0, int T, const float* alpha, cudaStream_t s);
cudaError_t launch_prefill_scan(const CacheView& c, int layer, int T0, int T, const float* alpha, cudaStream_t s);
cudaError_t launch_prefill_scatter(const CacheView& c, int layer, int T0, int T, const void* k, const void* v,
                                   cudaStream_t s);
// Tensor maps of the tcgen05 prefill attention: q [B*T, Hq, D] (box 64 x g x 128/g),
// k and v [B*T, Hkv, D] (box 64 x 1 x 128), kept copies [B*Hkv*max_pos, D] and
// window copies [B*Hkv*w, D] (box 64 x 64), all bf16 with the 128-byte
// swizzle.  `valid` is false when the shape is not covered.
struct PrefillMaps {
  CUtensorMap q, k, v, o, kept_k, kept_v, win_k, win_v;
  bool valid;
};
cudaError_t launch_prefill_attention(const CacheView& c, int T0, int T, const void* q, const void* k, const void* v,
                                     void* o, const PrefillMaps* maps, cudaStream_t s);
// pen: the training path's soft mode (every key before the window a prefix
// key from the input rows, scored with its penalty); null: DMS-masked prefill
// penmap: optional tensor map of pen as [B*Hkv rows, T] fp32 (box 64 x 1), when
// T % 4 == 0: the penalties then come by TMA with the V tiles
cudaError_t launch_prefill_attention_tc(const CacheView& c, int T0, int T, void* o, const PrefillMaps& maps,
                                        cudaStream_t s, const float* pen = nullptr,
                                        const CUtensorMap* penmap = nullptr);
cudaError_t launch_train_gate(long rows, int T, const float* alpha, const float* noise, float tau, float* prob,
                              float* hard, float* penalty, int num_sms, cudaStream_t s);
cudaError_t launch_decode_append(const CacheView& c, int layer, const void* k, const void* v, float* alpha,
                                 const DecideArgs* fused_decide, int num_sms, cudaStream_t s);
cudaError_t launch_decode_attention(const CacheView& c, int layer, const void* q, void* o,
                                    const CUtensorMap* kmap, const CUtensorMap* vmap, int num_sms,
                                    cudaStream_t s);
// Persistent split-K decode over all SMs; *taken is false (nothing launched)
// when the shape is outside what the kernel stages in shared memory.  `early`:
// the previous launch of this library on the stream was for another (cache,
// layer), so the kernel may read this layer's state before the previous
// kernels complete (programmatic dependent launch).
cudaError_t launch_decode_flat(const CacheView& c, int layer, const void* q, void* o, bool fused, const void* k,
                               const void* v, float* alpha, const DecideArgs* fused_decide, const CUtensorMap* kmap,
                               const CUtensorMap* vmap, cudaStream_t s, bool early, bool* taken);
// One cluster per (layer, b, h) of layers [layer, layer + nl): with nl > 1
// every input and output array holds the nl layers back to back (rows
// layer-major), and the fused step appends to all of them in one launch.
// Rows of the cluster decode kernel's TMA boxes for head dim D and page type.
int decode_cluster_box_rows(int D, bool fp8);
cudaError_t launch_decode_cluster(const CacheView& c, int layer, const void* q, void* o, bool fused, const void* k,
                                  const void* v, float* alpha, const DecideArgs* fused_decide, const CUtensorMap* kmap,
                                  const CUtensorMap* vmap, int num_sms, cudaStream_t s, bool early, int nl = 1);

// Programmatic dependent launch: let the next kernel of the stream start its
// prologue, and wait until every kernel this one depends on has completed.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// kern<<<grid, block, smem, s>>>(args...) as a programmatic dependent of the
// previous kernel on the stream: it may start while that kernel runs and
// reads nothing of its results before griddep_wait.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace dms
