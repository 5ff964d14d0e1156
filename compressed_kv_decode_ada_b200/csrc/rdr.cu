// rdr.cu -- the rate-distortion retention (RDR) controller: per token a
// residency decision and a precision tier b in {3,4,6,8} under a per-sequence
// byte budget, then the tier-homogeneous page layout of the plan.
//
// Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
// for Efficient Long-Context Inference", technical summary section 2.2 (a
// distortion surrogate from the angular error of the codes scaled by query
// and key magnitudes; residency and precision decided under a hard memory
// budget; protected states kept at the top tier; pages of one tier).  The
// readings of that section that this file implements:
//   - the decision unit is a token (its kv heads share a page, so a tier);
//   - D_t(b) = w_t eps_b, w_t = sum_h qn_h ||k_{t,h}||, eps_b = pi / (2^b
//     sqrt 12) (the RMS error of one uniformly coded angle), and an evicted
//     token costs w_t (eps = 1);
//   - a resident token's rate is H_kv (16 b + 1 + 256) bytes (codes, radius
//     byte, bf16 value row);
//   - protected tokens take b_max, the largest allowed tier.
// Solver: the Lagrangian relaxation -- each token minimises D_t(b) + lambda
// R(b) (equal costs: the larger b), and lambda is the smallest multiplier,
// found by doubling from 1 then bisection on [0, hi] (at most 100 halvings),
// whose total rate fits the budget.  Every decision is that of fp64 with the
// operations written out (__dmul_rn / __dadd_rn, no contraction), so the
// tiers, the multiplier and the rate are exact functions of the inputs; an
// fp32 filter with a proven margin (rdr_choose_fp32) takes the decisions
// fp64 would take, and hands every close one to fp64.
//
// Two kernels:
//   rdr_weights_kernel: w_t from the dense bf16 keys, HBM-bound (one read of
//     the keys, 8 bytes written per token), a full grid of warps;
//   rdr_plan_kernel: one thread-block cluster of kRdrCluster CTAs per
//     sequence; each pass evaluates every token at one lambda, the CTAs
//     exchange their per-tier counts through distributed shared memory, and
//     thread 0 of every CTA takes the same bisection step from the same
//     counts and publishes the next lambda to its CTA.  The bisection stops once
//     the midpoint equals an end of the bracket (the remaining halvings
//     cannot move it).  The last pass writes the tiers and packs the
//     resident tokens into pages: tiers ascending, tokens ascending within
//     a tier, each tier's group filling whole pages of 16 slots.
#include <cooperative_groups.h>

#include <cmath>

#include "spkv_common.cuh"

namespace cg = cooperative_groups;

namespace spkv {
namespace {

constexpr int kRdrCluster = 8;      // CTAs per sequence (portable cluster size)
constexpr int kRdrThreads = 1024;   // threads per plan CTA
constexpr int kRdrWarps = kRdrThreads / 32;
constexpr int kWThreads = 128;      // threads per weights CTA
constexpr int kWWarps = kWThreads / 32;
constexpr int kRowU4 = kD * 2 / 16;  // 16-byte chunks in one key row (16)
constexpr int kTileU4 = kRowU4 + 1;  // padded row stride in the staging tile
constexpr int kSmemTok = 16384;     // weights a plan CTA keeps in shared memory (fp64 + fp32: 192 KB)
constexpr float kMarginF = 1.0f - 0x1p-16f;  // fp32 decision margin (see rdr_choose_fp32)
constexpr int kMaxDoublings = 2000;
constexpr int kBisections = 100;

// ---------------------------------------------------------------- weights
struct WeightParams {
  const uint16_t *keys;       // [total_T, Hkv, 128] bf16
  const int32_t *seq_start;   // [B + 1]
  const float *qn;            // [B, Hkv]
  const uint8_t *protect;     // [total_T] or nullptr
  double *w;                  // [total_T] out: w_t, negated (sign bit) when protected
  int B, Hkv, tok_per_tile;
  int64_t total_T, tiles;
};

// Sequence of token t: the b with seq_start[b] <= t < seq_start[b + 1]
// (clamped into [0, B - 1]; tokens outside every range are never planned).
__device__ __forceinline__ int seq_of_token(const int32_t *seq_start, int B, int64_t t) {
  int lo = 0, hi = B;  // invariant: answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(seq_start + mid) <= t) lo = mid;
    else hi = mid;
  }
  return lo;
}

// |x| in fp64 for a bf16 bit pattern: for a normal bf16 the fp64 bits are
// the exponent rebiased (+ 1023 - 127) and the 7 fraction bits moved up;
// zero, subnormals, inf and NaN take the exact conversion.
__device__ __forceinline__ double bf16_abs_f64(uint32_t h16) {
  const uint32_t a = h16 & 0x7fffu;
  if (a >= 0x0080u && a < 0x7f80u) return __hiloint2double((int)((a << 13) + 0x38000000u), 0);
  return fabs(bf16_to_f64(a));
}

// One warp per tile of tok_per_tile tokens (tok_per_tile * Hkv <= 32 key
// rows): a coalesced copy of the tile's rows into shared memory (16-byte
// asynchronous copies, all sixteen of a lane in flight at once; rows padded
// to 272 bytes, so that the row-per-lane reads below are conflict-free), then
// lane r sums the squares of row r in ascending order (each square of a bf16
// value is exact in fp64, so n2 + x * x rounded once, an FMA, is the sum of
// the exact square), and the kv heads of a token are added in ascending
// order.
// Halfword-wise unsigned min / max of two words.
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__global__ void __launch_bounds__(kWThreads, 6) rdr_weights_kernel(const WeightParams p) {
  __shared__ uint4 tile[kWWarps][32 * kTileU4];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint4 *tl = tile[wid];
  const int64_t nwarps = (int64_t)gridDim.x * kWWarps;
  for (int64_t ti = (int64_t)blockIdx.x * kWWarps + wid; ti < p.tiles; ti += nwarps) {
    const int64_t t0 = ti * p.tok_per_tile;
    const int ntok = (int)min((int64_t)p.tok_per_tile, p.total_T - t0);
    const int rows = ntok * p.Hkv;
    const int nchunks = rows * kRowU4;
    const uint4 *src = reinterpret_cast<const uint4 *>(p.keys) + t0 * p.Hkv * kRowU4;
    // the tile: 16 asynchronous 16-byte copies per lane, all in flight at once
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = lane + 32 * i;
      if (c < nchunks)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(tl + (c >> 4) * kTileU4 + (c & 15))),
                     "l"(src + c)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    double pr = 0.0;  // qn_h * ||k_{t,h}|| of this lane's row
    const int h = lane % p.Hkv;
    const int64_t t = t0 + lane / p.Hkv;
    if (lane < rows) {
      const uint4 *row = tl + lane * kTileU4;
      // every element of the row a normal bf16 (exponent field 1..254)?
      uint32_t mn = 0xffffffffu, mx = 0u;
#pragma unroll 4
      for (int k = 0; k < kRowU4; ++k) {
        const uint4 q = row[k];
        const uint32_t a0 = q.x & 0x7fff7fffu, a1 = q.y & 0x7fff7fffu, a2 = q.z & 0x7fff7fffu, a3 = q.w & 0x7fff7fffu;
        mn = min_u16x2(mn, min_u16x2(min_u16x2(a0, a1), min_u16x2(a2, a3)));
        mx = max_u16x2(mx, max_u16x2(max_u16x2(a0, a1), max_u16x2(a2, a3)));
      }
      const bool normal = (mn & 0xffffu) >= 0x0080u && (mn >> 16) >= 0x0080u && (mx & 0xffffu) < 0x7f80u &&
                          (mx >> 16) < 0x7f80u;
      double n2 = 0.0;
      if (normal) {
        // |x| as fp64: exponent rebiased by 1023 - 127, fraction moved up
#pragma unroll 4
        for (int k = 0; k < kRowU4; ++k) {
          const uint4 q = row[k];
          const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const double x0 = __hiloint2double((int)((wv[e] & 0x7fffu) * 8192u + 0x38000000u), 0);
            const double x1 = __hiloint2double((int)(((wv[e] >> 3) & 0x0fffe000u) + 0x38000000u), 0);
            n2 = __fma_rn(x0, x0, n2);
            n2 = __fma_rn(x1, x1, n2);
          }
        }
      } else {
#pragma unroll 2
        for (int k = 0; k < kRowU4; ++k) {
          const uint4 q = row[k];
          const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const double x0 = bf16_abs_f64(wv[e] & 0xffffu), x1 = bf16_abs_f64(wv[e] >> 16);
            n2 = __fma_rn(x0, x0, n2);
            n2 = __fma_rn(x1, x1, n2);
          }
        }
      }
      const int b = seq_of_token(p.seq_start, p.B, t);
      pr = __dmul_rn((double)__ldg(p.qn + (int64_t)b * p.Hkv + h), __dsqrt_rn(n2));
    }
    // w_t = ((0 + pr_0) + pr_1) + ... over the token's lanes, in head order
    const int base = lane - h;
    double wt = 0.0;
    for (int hh = 0; hh < p.Hkv; ++hh) wt = __dadd_rn(wt, __shfl_sync(0xffffffffu, pr, min(base + hh, 31)));
    if (lane < rows && h == 0) {
      const bool prot = p.protect && p.protect[t];
      p.w[t] = prot ? -wt : wt;
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------- plan
struct PlanParams {
  const double *w;            // [total_T] signed weights (rdr_weights_kernel)
  const int32_t *seq_start;   // [B + 1]
  const double *budget;       // [B] bytes
  int B, imax, max_pages_out;
  int64_t total_T;
  uint32_t tier_mask;         // allowed tiers, bit i: b = {3,4,6,8}[i]
  double eps[kTiers];         // eps_b
  float epsf[kTiers];         // eps_b rounded to fp32
  double rate_d[kTiers];      // R(b), fp64
  uint64_t rate_u[kTiers];    // R(b), integer
  uint8_t *tier;              // [total_T] out: b, 0 = evicted
  int32_t *dst_pos;           // [total_T] out: packed position, -1 = evicted
  uint8_t *page_bits;         // [B, max_pages_out] out
  uint16_t *page_keep;        // [B, max_pages_out] out
  int32_t *n_pages;           // [B] out
  double *lambda, *rate, *dist;  // [B] out
  int32_t *status;            // [B] out (SPKV_RDR_* bits)
};

struct alignas(16) CtaCounts {
  uint4 n;        // tokens of this CTA at tier index 0..3
  uint32_t prot;  // protected tokens of this CTA
  uint32_t pad[3];
};

// The allowed tier index (0..3) minimising w eps_b + lambda R(b), -1 for
// eviction (cost w * 1 + lambda * 0); ties go to the larger b.  A negative
// w (sign bit) marks a protected token: b_max.  lam_r[i] = lambda R(b_i),
// lam_0 = lambda * 0 (NaN when lambda is infinite, so that every
// unprotected token is evicted then).
__device__ __forceinline__ int rdr_choose(double w, const PlanParams &p, const double (&lam_r)[kTiers],
                                          double lam_0) {
  if (signbit(w)) return p.imax;
  double bc = __dadd_rn(__dmul_rn(w, 1.0), lam_0);
  int best = -1;
#pragma unroll
  for (int i = 0; i < kTiers; ++i) {
    if (!((p.tier_mask >> i) & 1u)) continue;
    const double c = __dadd_rn(__dmul_rn(w, p.eps[i]), lam_r[i]);
    if (c <= bc) {
      bc = c;
      best = i;
    }
  }
  return best;
}

// The multiplier of one pass: lambda R(b_i) and lambda * 0 in fp64, and the
// fp32 copies of lambda R(b_i) for the fp32 filter (+inf for a tier that is
// not allowed, so that it never wins); the filter is off unless lambda is
// finite and every allowed lambda R(b_i) is zero or in [2^-100, 1e30].
struct PassLam {
  double r[kTiers], z;
  float rf[kTiers];
  bool fast;
};

__device__ __forceinline__ PassLam pass_lam(double lam, const PlanParams &p) {
  PassLam L;
  L.fast = isfinite(lam);
#pragma unroll
  for (int i = 0; i < kTiers; ++i) {
    L.r[i] = __dmul_rn(lam, p.rate_d[i]);
    const bool allowed = (p.tier_mask >> i) & 1u;
    L.rf[i] = allowed ? __double2float_rn(L.r[i]) : INFINITY;
    if (allowed) L.fast = L.fast && (L.r[i] == 0.0 || (L.r[i] >= 0x1p-100 && L.r[i] <= 1e30));
  }
  L.z = __dmul_rn(lam, 0.0);
  return L;
}

// The fp32 weight a token keeps for the filter: -1 when protected, |w|
// rounded to fp32 when |w| is 0 or in [2^-100, 1e30], NaN otherwise (no
// fp32 decision: every comparison with NaN fails).
__device__ __forceinline__ float filter_weight(double w) {
  if (signbit(w)) return -1.0f;
  return (w == 0.0 || (w >= 0x1p-100 && w <= 1e30)) ? __double2float_rn(w) : __int_as_float(0x7fc00000);
}

// rdr_choose first tried in fp32, without branches.  Each fp32 cost
// wf * eps_b + lambda R(b) (one FMA) is within 2^-22 of the real cost
// w eps_b + lambda R(b) (nonnegative terms; no underflow or overflow in the
// guarded range), and the fp64 cost of rdr_choose within 2^-51.9 of it.  If
// the fp32 minimum lies below every other fp32 cost by the factor 1 - 2^-16,
// the real costs differ by more than 2^-17 relative, so the fp64 costs are
// ordered the same way with no tie: the fp32 winner is the fp64 winner.
// need = true for anything closer (near-ties, equal costs) or unguarded:
// the caller then decides with rdr_choose.
struct FastDecision {
  int i;
  bool need;
};

__device__ __forceinline__ FastDecision rdr_choose_fp32(float wf, const PlanParams &p, const PassLam &L) {
  float best = wf, second = INFINITY;  // eviction: w * 1 + 0
  int bi = -1;
#pragma unroll
  for (int i = 0; i < kTiers; ++i) {
    const float c = __fmaf_rn(wf, p.epsf[i], L.rf[i]);
    const bool t = c <= best;
    second = t ? best : fminf(second, c);
    best = t ? c : best;
    bi = t ? i : bi;
  }
  const bool prot = wf < 0.0f;
  FastDecision d;
  d.i = prot ? p.imax : bi;
  d.need = !prot && !(L.fast && best < second * kMarginF);
  return d;
}

__global__ void __launch_bounds__(kRdrThreads, 1) rdr_plan_kernel(const PlanParams p) {
  static_assert(kRdrWarps == 32, "the CTA reductions give one warp's lane per warp");
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int seq = blockIdx.x / kRdrCluster;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  __shared__ CtaCounts part[2][kRdrCluster];  // every CTA's counts of one pass (double-buffered)
  __shared__ uint32_t wcnt[kRdrWarps][5];     // per-warp counts of one pass
  __shared__ uint4 wtot[2][kRdrWarps];        // packing: per-warp tier counts of one sweep step
  __shared__ double wdist[kRdrWarps];
  __shared__ double dpart[kRdrCluster];       // (rank 0) every CTA's distortion share

  const int64_t s0 = __ldg(p.seq_start + seq), s1 = __ldg(p.seq_start + seq + 1);
  cluster.sync();  // every CTA of the cluster is running before any remote access
  if (s0 < 0 || s1 < s0 || s1 > p.total_T) {  // (the same decision on every CTA)
    if (rank == 0 && tid == 0) {
      p.status[seq] = SPKV_RDR_BAD_RANGE;
      p.n_pages[seq] = 0;
      p.lambda[seq] = 0.0;
      p.rate[seq] = 0.0;
      p.dist[seq] = 0.0;
    }
    return;
  }
  const int64_t T = s1 - s0, chunk = (T + kRdrCluster - 1) / kRdrCluster;
  const int64_t c0 = s0 + min(T, chunk * rank), c1 = s0 + min(T, chunk * (rank + 1));
  const double budget = __ldg(p.budget + seq);
  int buf = 0;
  // this CTA's weights, read once (the first kSmemTok in shared memory; a
  // longer share reads the rest from global memory on every pass)
  extern __shared__ double wsm[];
  float *wfs = reinterpret_cast<float *>(wsm + kSmemTok);
  const int64_t nloc = c1 - c0;
  for (int64_t j = tid; j < min(nloc, (int64_t)kSmemTok); j += kRdrThreads) {
    const double w = __ldg(p.w + c0 + j);
    wsm[j] = w;
    wfs[j] = filter_weight(w);
  }
  __syncthreads();
  auto wget = [&](int64_t j) -> double { return j < kSmemTok ? wsm[j] : __ldg(p.w + c0 + j); };
  auto wfget = [&](int64_t j) -> float { return j < kSmemTok ? wfs[j] : filter_weight(__ldg(p.w + c0 + j)); };
  // The decision of token j: the fp32 filter, and rdr_choose where it abstains.
  auto decide = [&](int64_t j, const PassLam &L) -> int {
    const FastDecision d = rdr_choose_fp32(wfget(j), p, L);
    return d.need ? rdr_choose(wget(j), p, L.r, L.z) : d.i;
  };

  // One pass with the multiplier in L: this CTA's tokens are evaluated and
  // the CTAs' counts are exchanged (each CTA stores its record into every
  // CTA's part[buf]).  Returns the buffer the records are in.
  auto count_pass = [&](const PassLam &L) -> int {
    uint32_t c[kTiers] = {0u, 0u, 0u, 0u}, np = 0u;
    // groups of 4 tokens per thread decided without branches; a warp-wide
    // vote sends the (rare) abstentions to fp64.  The trip count is the same
    // for every thread of the CTA (the vote needs all 32 lanes).
    const int nl = (int)nloc;  // (< 2^31: seq_start is int32)
    for (int base = 0; base < nl; base += 4 * kRdrThreads) {
      const int j0 = base + tid;
      FastDecision d[4];
      bool valid[4];
      float wf[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + u * kRdrThreads;
        valid[u] = j < nl;
        wf[u] = valid[u] ? wfget(j) : 0.0f;
        d[u] = rdr_choose_fp32(wf[u], p, L);
        d[u].need = d[u].need && valid[u];
      }
      if (__any_sync(0xffffffffu, d[0].need || d[1].need || d[2].need || d[3].need)) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (d[u].need) d[u].i = rdr_choose(wget(j0 + u * kRdrThreads), p, L.r, L.z);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int t = 0; t < kTiers; ++t) c[t] += (valid[u] && d[u].i == t) ? 1u : 0u;
        np += (valid[u] && wf[u] < 0.0f) ? 1u : 0u;
      }
    }
    const uint32_t r0 = __reduce_add_sync(0xffffffffu, c[0]), r1 = __reduce_add_sync(0xffffffffu, c[1]);
    const uint32_t r2 = __reduce_add_sync(0xffffffffu, c[2]), r3 = __reduce_add_sync(0xffffffffu, c[3]);
    const uint32_t r4 = __reduce_add_sync(0xffffffffu, np);
    if (lane == 0) {
      wcnt[wid][0] = r0;
      wcnt[wid][1] = r1;
      wcnt[wid][2] = r2;
      wcnt[wid][3] = r3;
      wcnt[wid][4] = r4;
    }
    __syncthreads();
    if (wid == 0) {
      CtaCounts rec;
      rec.n.x = __reduce_add_sync(0xffffffffu, wcnt[lane][0]);
      rec.n.y = __reduce_add_sync(0xffffffffu, wcnt[lane][1]);
      rec.n.z = __reduce_add_sync(0xffffffffu, wcnt[lane][2]);
      rec.n.w = __reduce_add_sync(0xffffffffu, wcnt[lane][3]);
      rec.prot = __reduce_add_sync(0xffffffffu, wcnt[lane][4]);
      rec.pad[0] = rec.pad[1] = rec.pad[2] = 0u;
      if (lane < kRdrCluster) *cluster.map_shared_rank(&part[buf][rank], lane) = rec;
    }
    cluster.sync();
    const int used = buf;
    buf ^= 1;
    return used;
  };
  // Every CTA's counts of the pass whose records are in part[b], summed in rank order.
  auto totals = [&](int b, uint32_t (&tot)[kTiers], uint32_t &ptot) {
#pragma unroll
    for (int j = 0; j < kTiers; ++j) tot[j] = 0u;
    ptot = 0u;
#pragma unroll
    for (int r = 0; r < kRdrCluster; ++r) {
      const CtaCounts &q = part[b][r];
      tot[0] += q.n.x;
      tot[1] += q.n.y;
      tot[2] += q.n.z;
      tot[3] += q.n.w;
      ptot += q.prot;
    }
  };
  auto rate_of = [&](const uint32_t (&tot)[kTiers]) -> double {
    uint64_t r = 0;
#pragma unroll
    for (int j = 0; j < kTiers; ++j) r += (uint64_t)tot[j] * p.rate_u[j];
    return (double)r;
  };

  // ---- the multiplier.  Thread 0 of each CTA steps the search (the same
  // records give every CTA the same steps), in the oracle's order: lambda = 0;
  // if over budget and feasible, doubling from 1, then bisection on [lo, hi]
  // until the midpoint equals an end of the bracket (rate(lo) > budget and
  // rate(hi) <= budget throughout, so the remaining halvings would leave it
  // unchanged) or 100 halvings.  It publishes the next multiplier (with its
  // per-tier products) through shared memory: the scalar fp64 work is done
  // once per CTA, not by every thread.
  __shared__ PassLam ctl_L;
  __shared__ int ctl_go;
  double lam = 0.0, cur = 0.0, lo = 0.0, hi = 1.0;  // (thread 0)
  int st = 0, phase = 0, n = 0, it = 0;             // (thread 0)
  if (tid == 0) {
    ctl_L = pass_lam(0.0, p);
    ctl_go = 1;
  }
  __syncthreads();
  while (ctl_go) {  // (read after a __syncthreads: the same on every thread)
    const PassLam L = ctl_L;
    const int b = count_pass(L);
    if (tid == 0) {
      uint32_t tot[kTiers], ptot;
      totals(b, tot, ptot);
      const bool over = rate_of(tot) > budget;
      bool done = false, bisect = false;
      double next = 0.0;
      if (phase == 0) {  // lambda = 0
        if (!over) {
          done = true;
          lam = 0.0;
        } else if ((double)((uint64_t)ptot * p.rate_u[p.imax]) > budget) {
          done = true;  // protected tokens at b_max, every other one evicted
          st = SPKV_RDR_INFEASIBLE;
          lam = INFINITY;
        } else {
          phase = 1;
          hi = 1.0;
          n = 0;
          next = hi;
        }
      } else if (phase == 1) {  // doubling: cur = hi
        if (!over) {
          bisect = true;
        } else {
          hi *= 2.0;
          ++n;
          if (n < kMaxDoublings) next = hi;
          else bisect = true;
        }
        if (bisect) {
          phase = 2;
          lo = 0.0;
          it = 0;
        }
      } else {  // bisection: cur = the midpoint just evaluated
        if (over) lo = cur;
        else hi = cur;
        ++it;
        bisect = true;
      }
      if (bisect) {
        const double mid = __dmul_rn(0.5, __dadd_rn(lo, hi));
        if (it >= kBisections || mid == lo || mid == hi) {
          done = true;
          lam = hi;
        } else {
          next = mid;
        }
      }
      if (done) {
        ctl_go = 0;
        ctl_L = pass_lam(lam, p);
      } else {
        cur = next;
        ctl_L = pass_lam(next, p);
      }
    }
    __syncthreads();
  }

  // ---- the plan at lam: counts (and every CTA's counts, for the packing)
  const PassLam Lf = ctl_L;
  const int fb = count_pass(Lf);
  uint32_t tot[kTiers], ptot;
  totals(fb, tot, ptot);
  const double rate = tid == 0 ? rate_of(tot) : 0.0;  // (reported by thread 0 of rank 0)
  int64_t pstart[kTiers], npg[kTiers], total_pages = 0;
#pragma unroll
  for (int j = 0; j < kTiers; ++j) {
    pstart[j] = total_pages;
    npg[j] = ((int64_t)tot[j] + kPage - 1) / kPage;
    total_pages += npg[j];
  }
  const bool fits = total_pages <= (int64_t)p.max_pages_out;
  uint32_t cbase[kTiers] = {0u, 0u, 0u, 0u};  // this CTA's first rank within each tier
  for (int r = 0; r < rank; ++r) {
    const uint4 n = part[fb][r].n;
    cbase[0] += n.x;
    cbase[1] += n.y;
    cbase[2] += n.z;
    cbase[3] += n.w;
  }

  // ---- write sweep: tier, packed position (rank within the tier = tokens
  // of the tier before this one: earlier CTAs, earlier steps, earlier warps,
  // earlier lanes), and this CTA's share of the distortion
  const uint32_t lt_mask = (1u << lane) - 1u;
  double dl = 0.0;
  int step = 0;
  for (int64_t tb = c0; tb < c1; tb += kRdrThreads, ++step) {  // uniform over the CTA
    const int64_t t = tb + tid;
    const bool valid = t < c1;
    double w = 0.0;
    int i = -1;
    if (valid) {
      w = wget(t - c0);
      i = decide(t - c0, Lf);
    }
    uint32_t bal[kTiers];
#pragma unroll
    for (int j = 0; j < kTiers; ++j) bal[j] = __ballot_sync(0xffffffffu, i == j);
    if (lane == 0)
      wtot[step & 1][wid] = make_uint4(__popc(bal[0]), __popc(bal[1]), __popc(bal[2]), __popc(bal[3]));
    __syncthreads();
    // exclusive scan of the warps' counts: lane l holds warp l's counts
    const uint4 mine = wtot[step & 1][lane];
    uint32_t inc[kTiers] = {mine.x, mine.y, mine.z, mine.w};
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
      for (int j = 0; j < kTiers; ++j) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, inc[j], off);
        if (lane >= off) inc[j] += v;
      }
    }
    const uint32_t own[kTiers] = {mine.x, mine.y, mine.z, mine.w};
    uint32_t before[kTiers], all[kTiers];
#pragma unroll
    for (int j = 0; j < kTiers; ++j) {
      before[j] = __shfl_sync(0xffffffffu, inc[j] - own[j], wid);
      all[j] = __shfl_sync(0xffffffffu, inc[j], 31);
    }
    if (valid) {
      int32_t dpos = -1;
      uint8_t bits = 0;
      if (i >= 0) {
        bits = (uint8_t)bits_of_tier(i);
        uint32_t r = 0;
#pragma unroll
        for (int j = 0; j < kTiers; ++j)
          if (j == i) r = cbase[j] + before[j] + (uint32_t)__popc(bal[j] & lt_mask);
        int64_t ps = 0;
#pragma unroll
        for (int j = 0; j < kTiers; ++j)
          if (j == i) ps = pstart[j];
        if (fits) dpos = (int32_t)(ps * kPage + r);
      }
      p.tier[t] = bits;
      p.dst_pos[t] = dpos;
      double e = 1.0;
#pragma unroll
      for (int j = 0; j < kTiers; ++j)
        if (j == i) e = p.eps[j];
      dl = __dadd_rn(dl, __dmul_rn(fabs(w), e));
    }
#pragma unroll
    for (int j = 0; j < kTiers; ++j) cbase[j] += all[j];
  }

  // ---- the page layout (pages spread over the cluster's threads)
  if (fits) {
    for (int64_t pg = (int64_t)rank * kRdrThreads + tid; pg < total_pages; pg += (int64_t)kRdrCluster * kRdrThreads) {
      int j = 0;
#pragma unroll
      for (int k = 1; k < kTiers; ++k)
        if (pg >= pstart[k]) j = k;
      // (a tier with no pages has pstart equal to the next tier's: the last
      // such k wins, which is the tier that owns page pg)
      uint32_t n = 0;
      int64_t last = 0;
#pragma unroll
      for (int k = 0; k < kTiers; ++k)
        if (k == j) {
          n = tot[k] % kPage;
          last = pstart[k] + npg[k] - 1;
        }
      p.page_bits[(int64_t)seq * p.max_pages_out + pg] = (uint8_t)bits_of_tier(j);
      p.page_keep[(int64_t)seq * p.max_pages_out + pg] = (pg == last && n) ? (uint16_t)((1u << n) - 1u) : (uint16_t)0xffffu;
    }
  }

  // ---- the distortion: warps, then CTAs in rank order on rank 0
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dl = __dadd_rn(dl, __shfl_xor_sync(0xffffffffu, dl, off));
  if (lane == 0) wdist[wid] = dl;
  __syncthreads();
  if (wid == 0) {
    double v = wdist[lane];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
    if (lane == 0) *cluster.map_shared_rank(&dpart[rank], 0) = v;
  }
  cluster.sync();  // (the last remote access of the kernel)
  if (rank == 0 && tid == 0) {
    double d = 0.0;
    for (int r = 0; r < kRdrCluster; ++r) d = __dadd_rn(d, dpart[r]);
    p.dist[seq] = d;
    p.lambda[seq] = lam;
    p.rate[seq] = rate;
    p.n_pages[seq] = (int32_t)min(total_pages, (int64_t)INT32_MAX);
    p.status[seq] = st | (fits ? 0 : SPKV_RDR_PAGES);
  }
}

}  // namespace

int device_sm_count();

}  // namespace spkv

extern "C" size_t spkv_rdr_workspace_bytes(int64_t total_tokens) {
  if (total_tokens <= 0) return 16;
  return ((size_t)total_tokens * sizeof(double) + 15) / 16 * 16;
}

extern "C" spkv_status spkv_rdr_plan(const uint16_t *keys, const int32_t *seq_start, int32_t B, int64_t total_tokens,
                                     int32_t num_kv_heads, const float *q_norms, const uint8_t *protect,
                                     const double *budget_bytes, uint32_t tier_mask, int32_t max_pages_out,
                                     uint8_t *tier, int32_t *dst_pos, uint8_t *page_bits, uint16_t *page_keep,
                                     int32_t *n_pages, double *lambda, double *rate_bytes, double *distortion,
                                     int32_t *status, void *ws, size_t ws_bytes, void *stream) {
  using namespace spkv;
  const int Hkv = num_kv_heads;
  if (B < 0 || total_tokens < 0 || max_pages_out < 0 || Hkv < 1 || Hkv > 32) return SPKV_ERR_INVALID_ARG;
  if (tier_mask == 0u || tier_mask > 0xFu) return SPKV_ERR_INVALID_ARG;
  if (B == 0) return SPKV_OK;
  if (!seq_start || !q_norms || !budget_bytes || !n_pages || !lambda || !rate_bytes || !distortion || !status)
    return SPKV_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!keys || !tier || !dst_pos)) return SPKV_ERR_INVALID_ARG;
  if (max_pages_out > 0 && (!page_bits || !page_keep)) return SPKV_ERR_INVALID_ARG;
  if (((uintptr_t)keys & 15) || ((uintptr_t)page_keep & 1) || ((uintptr_t)ws & 15)) return SPKV_ERR_INVALID_ARG;
  if (!ws || ws_bytes < spkv_rdr_workspace_bytes(total_tokens)) return SPKV_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  double *w = (double *)ws;

  if (total_tokens > 0) {
    WeightParams wp;
    wp.keys = keys;
    wp.seq_start = seq_start;
    wp.qn = q_norms;
    wp.protect = protect;
    wp.w = w;
    wp.B = B;
    wp.Hkv = Hkv;
    wp.tok_per_tile = 32 / Hkv;
    wp.total_T = total_tokens;
    wp.tiles = (total_tokens + wp.tok_per_tile - 1) / wp.tok_per_tile;
    const int sms = device_sm_count();
    if (sms <= 0) return SPKV_ERR_CUDA;
    const int64_t want = (wp.tiles + kWWarps - 1) / kWWarps;
    const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    rdr_weights_kernel<<<grid, kWThreads, 0, st>>>(wp);
    if (cudaGetLastError() != cudaSuccess) return SPKV_ERR_CUDA;
  }

  PlanParams pp;
  pp.w = w;
  pp.seq_start = seq_start;
  pp.budget = budget_bytes;
  pp.B = B;
  pp.max_pages_out = max_pages_out;
  pp.total_T = total_tokens;
  pp.tier_mask = tier_mask;
  const double kPi = 3.14159265358979323846;
  pp.imax = 0;
  for (int i = 0; i < kTiers; ++i) {
    const int b = bits_of_tier(i);
    pp.eps[i] = kPi / (std::ldexp(1.0, b) * std::sqrt(12.0));
    pp.epsf[i] = (float)pp.eps[i];
    pp.rate_u[i] = (uint64_t)Hkv * (uint64_t)(16 * b + 1 + 256);
    pp.rate_d[i] = (double)pp.rate_u[i];
    if ((tier_mask >> i) & 1u) pp.imax = i;
  }
  pp.tier = tier;
  pp.dst_pos = dst_pos;
  pp.page_bits = page_bits;
  pp.page_keep = page_keep;
  pp.n_pages = n_pages;
  pp.lambda = lambda;
  pp.rate = rate_bytes;
  pp.dist = distortion;
  pp.status = status;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)B * kRdrCluster);
  cfg.blockDim = dim3(kRdrThreads);
  cfg.dynamicSmemBytes = (size_t)kSmemTok * (sizeof(double) + sizeof(float));
  if (cudaFuncSetAttribute(rdr_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)cfg.dynamicSmemBytes) != cudaSuccess)
    return SPKV_ERR_CUDA;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kRdrCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, rdr_plan_kernel, pp) != cudaSuccess) return SPKV_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}
