// spkv_common.cuh -- device helpers shared by the libspkv kernels (sm_100a).
//
// Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
// for Efficient Long-Context Inference", technical summary section 2.1
// (Angle-Domain Attention), 2.2 (tier-homogeneous pages) and 2.3 (paged,
// ragged KV substrate).  Layouts and numerical readings: include/spkv.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "spkv.h"

namespace spkv {

constexpr int kD = 128;       // head dimension
constexpr int kPage = 16;     // tokens per page
constexpr int kMaxB = 1024;   // largest batch the split kernels accept (2 CTAs / SM for every G)
constexpr int kTiers = 4;     // b in {3, 4, 6, 8}
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr int tier_of_bits(int b) { return b == 3 ? 0 : b == 4 ? 1 : b == 6 ? 2 : b == 8 ? 3 : -1; }
__host__ __device__ constexpr int bits_of_tier(int t) { return t == 0 ? 3 : t == 1 ? 4 : t == 2 ? 6 : 8; }
// Offset of tier t's 2^b-entry table inside a concatenated {3,4,6,8} table (344 entries).
__host__ __device__ constexpr int lut_off(int t) { return t == 0 ? 0 : t == 1 ? 8 : t == 2 ? 24 : 88; }
constexpr int kLutEntries = 344;
__host__ __device__ constexpr uint32_t rec_bytes(int b) { return 256u * (uint32_t)b + 16u; }

// ------------------------------------------------------------ small helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ double bf16_to_f64(uint32_t h16) {
  double x = (double)__uint_as_float(h16 << 16);
  return x == 0.0 ? 0.0 : x;  // -0 -> +0
}

// d = a * b + c on a pair of fp32 lanes (one f32x2 instruction on sm_100a).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void set_err(uint32_t *err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

// ------------------------------------------------------------ mbarrier / bulk copy
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase `parity`; the answer may be consumed much later.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Like mbar_wait_bounded, for a thread that is expected to wait long (a
// producer ahead of its consumers): it sleeps in try_wait between checks.
__device__ __forceinline__ bool mbar_wait_sleepy(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > 1000000000ull) {
      *abort = 1;
      set_err(err, SPKV_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// Wait for phase `parity` of *bar to complete, giving up after ~1 s of wall
// time (or as soon as *abort is set by another warp).  On a timeout it sets
// SPKV_DEVERR_TIMEOUT and *abort, and returns false; callers then carry on
// with the same control flow (so every barrier is still reached) but the
// results of this call are flagged as invalid.
// sleep_ns > 0 backs off between polls (for waiters off the critical path).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                  uint32_t *err, uint32_t sleep_ns = 0,
                                                  uint64_t limit_ns = 1000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (sleep_ns) __nanosleep(sleep_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if ((it & 63u) == 63u && globaltimer_ns() - t0 > limit_ns) {
      *abort = 1;
      set_err(err, SPKV_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// 1-D bulk copy global -> this CTA's shared memory; completion is counted in
// bytes on *bar.  Both addresses 16-byte aligned, bytes a multiple of 16.
// (No cluster multicast anywhere in this library.)
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled TMA load (box of the tensor map at element coordinates (x, y, z))
// into this CTA's shared memory, completion counted on *bar.  No multicast.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) accesses of the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------ work partition
// The (page, kv head) units of a batch are numbered u = P[b] + h * np_b + j
// (sequence-major, then kv head, then page), where np_b = ceil(ctx_b / 16)
// and P is the exclusive prefix sum of np_b * H_kv (W = P[B] units).  A kv row
// r = b * H_kv + h holds units [rs(r), rs(r + 1)).  Split c of C owns a
// contiguous range of units, cut at equal steps of a weighted position
//   f(u) = u + kRowCostUnits * r(u),
// i.e. every row boundary costs kRowCostUnits units: a split that crosses one
// runs a second segment (query preparation, a warp barrier, partials) and gets
// that many fewer pages.  With F = W + kRowCostUnits * B * H_kv and
// t_c = floor(c F / C), split c begins at the first unit u with f(u) >= t_c.
// Each (split, kv-head row bh) intersection is a segment whose partial result
// goes to workspace slot c + bh (unique because both indices only grow along
// the unit order).
constexpr int64_t kRowCostUnits = 20;

struct Partition {
  const int32_t *P;
  int B, Hkv, C;
  int64_t W, F;
  __device__ __forceinline__ Partition(const int32_t *P_, int B_, int Hkv_, int C_)
      : P(P_), B(B_), Hkv(Hkv_), C(C_) {
    W = P[B];
    F = W + kRowCostUnits * (int64_t)B * Hkv;
  }
  // weighted start of sequence b: f of its first unit (rows before it: b * Hkv)
  __device__ __forceinline__ int64_t seq_f(int b) const { return (int64_t)P[b] + kRowCostUnits * (int64_t)b * Hkv; }
  __device__ __forceinline__ int64_t target(int c) const { return (F * (int64_t)c) / C; }
  // first unit of split c (begin(C) = W): the first u with f(u) >= t_c
  __device__ __forceinline__ int64_t begin(int c) const {
    if (c <= 0) return 0;
    if (c >= C) return W;
    const int64_t t = target(c);
    int lo = 0, hi = B - 1;  // last sequence b with seq_f(b) <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (seq_f(mid) <= t) lo = mid;
      else hi = mid - 1;
    }
    const uint32_t np = (uint32_t)(P[lo + 1] - P[lo]) / (uint32_t)Hkv;
    const uint32_t d = (uint32_t)(t - seq_f(lo));  // < Hkv (np + k) + k, fits 32 bits
    uint32_t h = d / (np + (uint32_t)kRowCostUnits);
    if (h > (uint32_t)Hkv - 1u) h = (uint32_t)Hkv - 1u;
    const int64_t rs = (int64_t)P[lo] + (int64_t)h * np;
    const int64_t u = rs + (int64_t)(d - h * (np + (uint32_t)kRowCostUnits));
    const int64_t re = rs + np;
    return u < re ? u : re;  // t in the gap after the row: the next row's first unit
  }
  // the split whose units contain unit u of kv row r: the last c with t_c <= f(u)
  __device__ __forceinline__ int64_t split_of(int64_t u, int64_t r) const {
    const int64_t f = u + kRowCostUnits * r;
    return ((f + 1) * C - 1) / F;
  }
  // For the splits [cf, cl] that meet one row (cf = split_of(first unit),
  // cl = split_of(last unit)): cf and cl hold units of the row, and a split
  // in between begins inside the row at a + t_c - f(a), so it holds units
  // iff t_c < t_{c+1}.
  __device__ __forceinline__ bool live_in_row(int64_t c, int64_t cf, int64_t cl) const {
    return c == cf || c == cl || target((int)c) < target((int)c + 1);
  }
};

// Pages of a sequence, validated against max_ctx and max_pages.
__device__ __forceinline__ int seq_pages(int ctx, int max_ctx, int max_pages, uint32_t *err) {
  if (ctx < 0 || ctx > max_ctx || ctx > max_pages * kPage) {
    if (ctx != 0) set_err(err, SPKV_DEVERR_CTX);
    return 0;
  }
  return (ctx + kPage - 1) / kPage;
}

// Block-wide exclusive prefix of np_b * Hkv into P[0..B] (P[B] = W), computed
// by all `nthreads` threads of the block (a multiple of 32, <= 1024).
__device__ __forceinline__ void build_prefix(const int32_t *ctx_lens, int B, int Hkv, int max_ctx, int max_pages,
                                             uint32_t *err, int32_t *P, int32_t *scratch32, int tid,
                                             int nthreads) {
  const int per = (B + nthreads - 1) / nthreads;
  const int b0 = tid * per;
  int32_t local = 0;
  for (int i = 0; i < per; ++i) {
    const int b = b0 + i;
    if (b < B) {
      const int np = seq_pages(ctx_lens[b], max_ctx, max_pages, err);
      P[b] = np * Hkv;  // temporarily the count
      local += np * Hkv;
    }
  }
  // exclusive scan of `local` across the block
  const int lane = tid & 31, wid = tid >> 5, nw = nthreads >> 5;
  int32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scratch32[wid] = incl;
  __syncthreads();
  if (tid == 0) {
    int32_t run = 0;
    for (int w = 0; w < nw; ++w) {
      int32_t v = scratch32[w];
      scratch32[w] = run;
      run += v;
    }
    scratch32[nw] = run;
  }
  __syncthreads();
  int32_t run = scratch32[wid] + incl - local;
  for (int i = 0; i < per; ++i) {
    const int b = b0 + i;
    if (b < B) {
      const int32_t cnt = P[b];
      P[b] = run;
      run += cnt;
    }
  }
  if (tid == 0) P[B] = scratch32[nw];
  __syncthreads();
}

// Largest b with P[b] <= u (P non-decreasing, P[0] = 0, u < P[B]).
__device__ __forceinline__ int find_seq(const int32_t *P, int B, int64_t u) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)P[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------ exact code decisions
// Squared cosines of the cell edges, fp64, for the four tiers concatenated:
//   polar   edge k of b bits: theta = k pi / 2^b      -> pol_c2[lut_off(t) + k]
//   azimuth edge k of b bits: theta = k 2 pi / 2^b    -> az_c2[lut_off(t) + k]
// Computed as (1 + cos 2 theta) / 2 so that the edges at multiples of pi/4,
// the only ones a bf16 input can hit exactly, get the exact values 1, 1/2, 0:
// an exact tie is then decided exactly (to the upper cell).
// half_signed: the polar entries of the lower half of [0, pi] (k < 2^(b-1))
// as above and those of the upper half negated, -cos^2 (the bulk encoder's
// one-comparison search, polar_code_half<BITS, true>).
__device__ __forceinline__ void build_edge_tables(double *pol_c2, double *az_c2, int tid, int nthreads,
                                                  bool half_signed = false) {
  for (int i = tid; i < kLutEntries; i += nthreads) {
    const int t = i < 8 ? 0 : i < 24 ? 1 : i < 88 ? 2 : 3;
    const int b = bits_of_tier(t), k = i - lut_off(t);
    const double c2 = 0.5 * (1.0 + cospi((double)(2 * k) / (double)(1 << b)));
    pol_c2[i] = half_signed && 2 * k >= (1 << b) ? -c2 : c2;
    az_c2[i] = 0.5 * (1.0 + cospi((double)(4 * k) / (double)(1 << b)));
  }
}

// phi >= theta_k for a polar angle, given x = x_i, S = S_i = sum_{j>=i} x_j^2
// (S > 0), the edge's squared cosine c2 and whether its cosine is >= 0:
// phi >= theta  <=>  cos(phi) = x / sqrt(S) <= cos(theta).
__device__ __forceinline__ bool polar_reaches(double x, double S, double c2, bool cos_nonneg) {
  const double x2 = x * x, rhs = S * c2;
  return cos_nonneg ? (x <= 0.0 || x2 <= rhs) : (x < 0.0 && x2 >= rhs);
}

// floor(phi 2^b / pi) clamped to 2^b - 1 for phi = atan2(sqrt(S_{i+1}), x_i),
// by binary search over the edges (the largest edge the angle reaches).
template <int BITS>
__device__ __forceinline__ int polar_code(double x, double S, const double *c2) {
  if (S == 0.0) return 0;  // atan2(0, 0) = 0
  int lo = 0, hi = (1 << BITS) - 1;
#pragma unroll
  for (int it = 0; it < BITS; ++it) {
    const int mid = (lo + hi + 1) >> 1;
    if (polar_reaches(x, S, c2[mid], mid <= (1 << (BITS - 1)))) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// floor(phi 2^b / 2 pi) for the azimuth phi = atan2(z, a) taken in [0, 2 pi),
// with a = x_126, z = x_127, S = a^2 + z^2.  z >= 0: phi in [0, pi] and the
// polar test applies to the edges k <= 2^(b-1); z < 0: phi in (pi, 2 pi), every
// edge k <= 2^(b-1) is reached and above it phi >= theta_k <=> a >= rho cos theta_k.
template <int BITS>
__device__ __forceinline__ int azimuth_code(double a, double z, double S, const double *c2) {
  if (S == 0.0) return 0;
  constexpr int H = 1 << (BITS - 1), Q = 1 << (BITS - 2);
  int lo = 0, hi = (1 << BITS) - 1;
#pragma unroll
  for (int it = 0; it < BITS; ++it) {
    const int k = (lo + hi + 1) >> 1;
    bool reach;
    if (z >= 0.0) {
      reach = (k <= H) && polar_reaches(a, S, c2[k], k <= Q);
    } else if (k <= H) {
      reach = true;
    } else {
      const double a2 = a * a, rhs = S * c2[k];
      reach = (k >= 3 * Q) ? (a >= 0.0 && a2 >= rhs) : (a >= 0.0 || a2 <= rhs);
    }
    if (reach) lo = k; else hi = k - 1;
  }
  return lo;
}

// The four fp64 inputs of one warp lane (x_{4l..4l+3}) and the suffix sums
// S_i = sum_{j >= i} x_j^2 (squares of bf16 values are exact in fp64).
__device__ __forceinline__ void lane_suffix_sums(uint2 raw, int lane, double (&x)[4], double (&S)[4]) {
  x[0] = bf16_to_f64(raw.x & 0xffffu);
  x[1] = bf16_to_f64(raw.x >> 16);
  x[2] = bf16_to_f64(raw.y & 0xffffu);
  x[3] = bf16_to_f64(raw.y >> 16);
  S[3] = x[3] * x[3];
  S[2] = x[2] * x[2] + S[3];
  S[1] = x[1] * x[1] + S[2];
  S[0] = x[0] * x[0] + S[1];
  double incl = S[0];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double v = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += v;
  }
  double after = __shfl_down_sync(0xffffffffu, incl, 1);
  if (lane == 31) after = 0.0;
#pragma unroll
  for (int k = 0; k < 4; ++k) S[k] += after;
}

// Angle codes of the lane's four fields a = 4 lane + k at b = BITS bits
// (field 126 is the azimuth, field 127 the zero padding).
template <int BITS>
__device__ __forceinline__ void lane_codes(const double (&x)[4], const double (&S)[4], double x127, int lane,
                                           const double *pol_c2, const double *az_c2, int (&c)[4]) {
  const double *pc2 = pol_c2 + lut_off(tier_of_bits(BITS));
  const double *ac2 = az_c2 + lut_off(tier_of_bits(BITS));
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int a = 4 * lane + k;
    if (a < 126) c[k] = polar_code<BITS>(x[k], S[k], pc2);
    else if (a == 126) c[k] = azimuth_code<BITS>(x[k], x127, S[k], ac2);
    else c[k] = 0;
  }
}

}  // namespace spkv
