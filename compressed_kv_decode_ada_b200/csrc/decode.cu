// decode.cu -- paged decode attention over spherical codes (ADA) and the two
// comparison paths (dense bf16 keys; decompress-then-dot), sm_100a.
//
// Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
// for Efficient Long-Context Inference", technical summary section 2.1:
// during the decode hot loop the attention kernel computes the logits straight
// from the quantised radius and the packed angle codes,
//     logit ~= ||q|| * r~ * f_b(c_q, c_k)   (here divided by sqrt(d)),
// where f_b is a fused kernel operation giving the cosine similarity from the
// angle codes, and no dense key vector is ever materialised in HBM.  Section
// 2.2: pages are tier-homogeneous, so the kernel streams each page once,
// guided by its header.  The problem statement of the same summary names the
// "decompress, then dot product" path that ADA replaces.
//
// Kernel design (B200):
//  * Work = (page, kv head) units of the whole ragged batch, numbered
//    sequence-major; split c of C owns a contiguous, equal share (balanced for
//    any mix of context lengths), so C = SMs x resident CTAs is one full wave.
//  * CTA = 1 producer warp + 4 consumer warps.  The producer resolves block
//    table -> page header -> record address and streams each unit's code
//    record (256 b + 16 bytes) and its 4 KB value page into a shared-memory
//    ring with 1-D bulk copies (cp.async.bulk, mbarrier completion).  Consumer
//    warp w takes units w, w+4, ... and keeps its own online-softmax state.
//  * f_b: lane = (slot t, half of the angle chain).  Each lane decodes 64
//    angle codes of its slot, looks up (cos, sin) of the cell midpoint in a
//    shared-memory table and runs the prefix product of sines
//        u_j = (prod_{i<j} sin phi_i) cos phi_j,
//    accumulating <u_q, u_k> for the G query heads of the kv head on CUDA
//    cores (f32x2 FMAs).  The two halves are joined by
//        f = A + (prod_{i<=64} sin phi_i) * B.
//    The key's unit vector lives only in registers.
//  * Online softmax in the log2 domain; P.V with lane = 4 value dims.
//  * Per segment the 4 warps' states are merged and written as one partial
//    (m, l, acc[128]) per query head; a second kernel merges the partials.
#include <cuda_bf16.h>

#include <type_traits>

#include "spkv_common.cuh"

namespace spkv {

spkv_status check_cache(const spkv_cache *c);
int device_sm_count();

namespace {

constexpr int kNCW = 4;                      // consumer warps
constexpr int kThreads = (kNCW + 1) * 32;    // + producer warp
#define kNegInf (-__int_as_float(0x7f800000))

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// ----------------------------------------------------------------- layout
template <bool ADA, int G>
struct Layout {
  static constexpr int NST = ADA ? 12 : 8;                    // ring stages (3 or 2 per consumer warp)
  static constexpr int STAGE = ADA ? (4096 + 2064) : 8192;    // V page + largest record | K + V page
  static constexpr int REC_OFF = 4096;                        // ADA: record after the V page
  static constexpr int KV_OFF = 4096;                         // dense: V after the K page
  static constexpr int QT_HALF = ADA ? (64 * G + 4) : 8 * (8 * G + 4);  // floats, +16 B skew
  static constexpr int QT_TIER = 2 * QT_HALF;
  static constexpr int QT_FLOATS = (ADA ? kTiers : 1) * QT_TIER;
  static constexpr int CMB = 132;                             // m, l, pad, pad, acc[128]
  static constexpr int CMB_FLOATS = kNCW * G * CMB;
  static constexpr int UNION_FLOATS = QT_FLOATS > CMB_FLOATS ? QT_FLOATS : CMB_FLOATS;
  static constexpr int PBUF_FLOATS = kNCW * kPage * G * 2;

  static constexpr int off_stage = 0;
  static constexpr int off_lut = off_stage + NST * STAGE;
  static constexpr int lut_bytes = ADA ? 2 * kLutEntries * 8 : 0;
  static constexpr int off_union = off_lut + lut_bytes;
  static constexpr int off_pbuf = off_union + UNION_FLOATS * 4;
  static constexpr int off_sc = off_pbuf + PBUF_FLOATS * 4;   // G scales + L_h + Delta_h
  static constexpr int off_bar = off_sc + ((G + 2) * 4 + 15) / 16 * 16;
  static constexpr int off_meta = off_bar + 2 * NST * 8;
  static constexpr int off_misc = off_meta + NST * 16;       // abort flag + scan scratch
  static constexpr int off_P = off_misc + 16 + 36 * 4;
  static size_t bytes(int B) { return (size_t)off_P + (size_t)(B + 1) * 4 + 16; }
};

struct SplitParams {
  const uint8_t *arena;
  uint64_t arena_bytes;
  const spkv_page_hdr *hdr;
  const float *rad_lo, *rad_step;
  const uint16_t *k_pages;  // dense path only
  const uint16_t *v_pages;
  const uint16_t *keep;
  uint32_t *err;
  int Hkv, num_pages;
  const uint16_t *q;
  int B, Hq;
  const int32_t *block_table;
  int max_pages;
  const int32_t *ctx_lens;
  int max_ctx;
  float *ws;
};

// Stage metadata written by the producer, read by the consumer.
struct StageMeta {
  int valid;   // 0: skip this unit (bad page / header / record)
  int bits;    // ADA tier bit width
  int ntok;    // valid slots in the page (1..16)
  uint32_t live;  // keep-mask bits restricted to the first ntok slots
};

// ----------------------------------------------------------- ADA pieces
// (cos, sin) of the cell midpoints, fp32: polar (c + 1/2) pi / 2^b and azimuth
// (c + 1/2) 2 pi / 2^b, for the four tiers concatenated.
__device__ __forceinline__ void build_luts(float2 *lpol, float2 *laz, int tid, int nthreads) {
  for (int i = tid; i < kLutEntries; i += nthreads) {
    const int t = i < 8 ? 0 : i < 24 ? 1 : i < 88 ? 2 : 3;
    const int b = bits_of_tier(t), c = i - lut_off(t);
    float s, co;
    sincospif(((float)c + 0.5f) / (float)(1 << b), &s, &co);
    lpol[i] = make_float2(co, s);
    sincospif(((float)c + 0.5f) / (float)(1 << (b - 1)), &s, &co);
    laz[i] = make_float2(co, s);
  }
}

// One warp: the coded query (section 2.1's c_theta^q; the query is coded at
// each tier's b) -> decoded unit vector per tier, written to
// qt[tier * QT_TIER + half * QT_HALF + (pair * G + g) * 2 + e] for slot
// a = 64 half + 2 pair + e.  Angle codes are decided in fp64.  Returns ||q||.
template <int G, int QT_HALF>
__device__ float ada_qprep_row(const uint16_t *qrow, int g, const float2 *lpol, const float2 *laz, float *qt,
                               int lane) {
  const uint2 raw = *reinterpret_cast<const uint2 *>(qrow + 4 * lane);
  const double x[4] = {bf16_to_f64(raw.x & 0xffffu), bf16_to_f64(raw.x >> 16), bf16_to_f64(raw.y & 0xffffu),
                       bf16_to_f64(raw.y >> 16)};
  double S[4];
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
  const double x127 = __shfl_sync(0xffffffffu, x[3], 31);
  const double nextS0 = __shfl_down_sync(0xffffffffu, S[0], 1);
  double phi[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int a = 4 * lane + k;
    const double Snext = k < 3 ? S[k + 1] : (lane == 31 ? 0.0 : nextS0);
    if (a < 126) {
      phi[k] = atan2(sqrt(Snext), x[k]);
    } else if (a == 126) {
      double v = atan2(x127, x[k]);
      if (v < 0.0) v += 2.0 * 3.14159265358979323846;
      phi[k] = v;
    } else {
      phi[k] = 0.0;
    }
  }
  const double qn = sqrt(__shfl_sync(0xffffffffu, S[0], 0));
#pragma unroll
  for (int ti = 0; ti < kTiers; ++ti) {
    const int b = bits_of_tier(ti);
    const int top = (1 << b) - 1;
    float2 cs[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int a = 4 * lane + k;
      if (a < 126) {
        const int c = min(top, (int)floor(phi[k] * (double)(1 << b) / 3.14159265358979323846));
        cs[k] = lpol[lut_off(ti) + c];
      } else if (a == 126) {
        const int c = min(top, (int)floor(phi[k] * (double)(1 << b) / (2.0 * 3.14159265358979323846)));
        cs[k] = laz[lut_off(ti) + c];
      } else {
        cs[k] = make_float2(1.0f, 0.0f);  // padding field: u_127 = product of all sines
      }
    }
    const float pl1 = cs[0].y, pl2 = pl1 * cs[1].y, pl3 = pl2 * cs[2].y, lane_prod = pl3 * cs[3].y;
    float inc = lane_prod;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc *= v;
    }
    float E = __shfl_up_sync(0xffffffffu, inc, 1);
    if (lane == 0) E = 1.0f;
    const float u[4] = {E * cs[0].x, E * pl1 * cs[1].x, E * pl2 * cs[2].x, E * pl3 * cs[3].x};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int a = 4 * lane + k;
      const int half = a >> 6, s = a & 63;
      qt[ti * 2 * QT_HALF + half * QT_HALF + ((s >> 1) * G + g) * 2 + (s & 1)] = u[k];
    }
  }
  return (float)qn;
}

template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&W)[2 * BITS], int a) {
  const int bit = a * BITS, w = bit >> 5, sh = bit & 31;
  uint32_t v;
  if (sh + BITS <= 32) v = W[w] >> sh;
  else v = __funnelshift_r(W[w], W[w + 1], sh);
  return v & ((1u << BITS) - 1u);
}

// f_b for the 16 slots of one record and the G heads (valid on lanes 0..15).
template <int BITS, int G, int QT_HALF>
__device__ __forceinline__ void ada_page_f(const uint8_t *rec, const float *qt, const float2 *lpol,
                                           const float2 *laz, int lane, float (&f)[G]) {
  const int t = lane & 15, half = lane >> 4;
  uint32_t W[2 * BITS];
  if constexpr ((BITS & 1) == 0) {
#pragma unroll
    for (int k = 0; k < BITS / 2; ++k) {
      const uint4 v = *reinterpret_cast<const uint4 *>(rec + ((half * (BITS / 2) + k) * 16 + t) * 16);
      W[4 * k + 0] = v.x;
      W[4 * k + 1] = v.y;
      W[4 * k + 2] = v.z;
      W[4 * k + 3] = v.w;
    }
  } else {
    static_assert(BITS == 3, "odd widths other than 3 are not supported");
    const uint4 A = *reinterpret_cast<const uint4 *>(rec + ((half + 0) * 16 + t) * 16);
    const uint4 Bv = *reinterpret_cast<const uint4 *>(rec + ((half + 1) * 16 + t) * 16);
    W[0] = half ? A.z : A.x;
    W[1] = half ? A.w : A.y;
    W[2] = half ? Bv.x : A.z;
    W[3] = half ? Bv.y : A.w;
    W[4] = half ? Bv.z : Bv.x;
    W[5] = half ? Bv.w : Bv.y;
  }
  const float *qh = qt + half * QT_HALF;
  const float2 *l62 = half ? laz : lpol;
  float P = 1.0f;
  float2 acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
#pragma unroll
  for (int a = 0; a < 64; a += 2) {
    const uint32_t c0 = code_at<BITS>(W, a), c1 = code_at<BITS>(W, a + 1);
    float2 e0, e1;
    if (a == 62) {
      e0 = l62[c0];
      const float2 t1 = lpol[half ? 0u : c1];
      e1 = make_float2(half ? 1.0f : t1.x, half ? 0.0f : t1.y);
    } else {
      e0 = lpol[c0];
      e1 = lpol[c1];
    }
    const float u0 = P * e0.x;
    P *= e0.y;
    const float u1 = P * e1.x;
    P *= e1.y;
    const float2 uu = make_float2(u0, u1);
    const float *qp = qh + (a >> 1) * G * 2;
    if constexpr (G == 1) {
      const float2 q2 = *reinterpret_cast<const float2 *>(qp);
      acc[0] = ffma2(uu, q2, acc[0]);
    } else {
#pragma unroll
      for (int g = 0; g < G; g += 2) {
        const float4 q4 = *reinterpret_cast<const float4 *>(qp + 2 * g);
        acc[g] = ffma2(uu, make_float2(q4.x, q4.y), acc[g]);
        acc[g + 1] = ffma2(uu, make_float2(q4.z, q4.w), acc[g + 1]);
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float A = acc[g].x + acc[g].y;
    const float Bh = __shfl_down_sync(0xffffffffu, A, 16);
    f[g] = fmaf(P, Bh, A);
  }
}

// --------------------------------------------------------- dense pieces
// q (scaled by log2(e)/sqrt(d)) as fp32 in [half][chunk][g][8] with a 16-byte
// skew per chunk so that lanes reading rotated chunks hit distinct banks.
template <int G, int QT_HALF>
__device__ void dense_qprep_row(const uint16_t *qrow, int g, float *qt, int lane) {
  const uint2 raw = *reinterpret_cast<const uint2 *>(qrow + 4 * lane);
  const float s = kLog2e * 0.08838834764831845f;  // log2(e) / sqrt(128)
  const float v[4] = {bf16lo(raw.x) * s, bf16hi(raw.x) * s, bf16lo(raw.y) * s, bf16hi(raw.y) * s};
  const int half = lane >> 4, chunk = (lane & 15) >> 1, off = (lane & 1) * 4;
  float *dst = qt + half * QT_HALF + chunk * (8 * G + 4) + g * 8 + off;
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = v[i];
}

template <int G, int QT_HALF>
__device__ __forceinline__ void dense_page_logits(const uint8_t *kpage, const float *qt, int lane, float (&l2)[G]) {
  const int t = lane & 15, half = lane >> 4;
  float acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = 0.f;
  const uint8_t *krow = kpage + t * 256 + half * 128;
  const float *qh = qt + half * QT_HALF;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int ch = (i + t) & 7;
    const uint4 kw = *reinterpret_cast<const uint4 *>(krow + ch * 16);
    const float k[8] = {bf16lo(kw.x), bf16hi(kw.x), bf16lo(kw.y), bf16hi(kw.y),
                        bf16lo(kw.z), bf16hi(kw.z), bf16lo(kw.w), bf16hi(kw.w)};
    const float *qc = qh + ch * (8 * G + 4);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 qa = *reinterpret_cast<const float4 *>(qc + g * 8);
      const float4 qb = *reinterpret_cast<const float4 *>(qc + g * 8 + 4);
      float2 s2 = make_float2(0.f, 0.f);
      s2 = ffma2(make_float2(qa.x, qa.y), make_float2(k[0], k[1]), s2);
      s2 = ffma2(make_float2(qa.z, qa.w), make_float2(k[2], k[3]), s2);
      s2 = ffma2(make_float2(qb.x, qb.y), make_float2(k[4], k[5]), s2);
      s2 = ffma2(make_float2(qb.z, qb.w), make_float2(k[6], k[7]), s2);
      acc[g] += s2.x + s2.y;
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) l2[g] = acc[g] + __shfl_down_sync(0xffffffffu, acc[g], 16);
}

// ------------------------------------------------------ split kernel
template <bool ADA, int G>
__global__ void __launch_bounds__(kThreads) split_kernel(const SplitParams p) {
  using Ly = Layout<ADA, G>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *stages = smem + Ly::off_stage;
  float2 *lpol = reinterpret_cast<float2 *>(smem + Ly::off_lut);
  float2 *laz = lpol + kLutEntries;
  float *uni = reinterpret_cast<float *>(smem + Ly::off_union);
  float *pbuf_all = reinterpret_cast<float *>(smem + Ly::off_pbuf);
  float *sc = reinterpret_cast<float *>(smem + Ly::off_sc);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + Ly::off_bar);
  uint64_t *empty = full + Ly::NST;
  StageMeta *meta = reinterpret_cast<StageMeta *>(smem + Ly::off_meta);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Ly::off_misc);
  int32_t *scratch = reinterpret_cast<int32_t *>(smem + Ly::off_misc + 16);
  int32_t *P = reinterpret_cast<int32_t *>(smem + Ly::off_P);

  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int C = gridDim.x, c = blockIdx.x;

  build_prefix(p.ctx_lens, p.B, p.Hkv, p.max_ctx, p.max_pages, p.err, P, scratch, tid, kThreads);
  const int64_t W = P[p.B];
  const int64_t u0 = split_begin(W, C, c), u1 = split_begin(W, C, c + 1);
  if (u0 >= u1) return;  // uniform across the block

  if (tid == 0) {
    for (int s = 0; s < Ly::NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if constexpr (ADA) build_luts(lpol, laz, tid, kThreads);
  __syncthreads();

  const int n_units = (int)(u1 - u0);

  if (wid == kNCW) {
    // =========================== producer warp ===========================
    // Metadata of a batch of 32 units is fetched by the 32 lanes in two
    // dependent rounds (block table, then header / mask), one batch ahead.
    struct A_ {
      int pid, ntok, h, ok;
    };
    struct B_ {
      uint32_t off16;
      int bits;
      uint32_t keep;
    };
    auto phaseA = [&](int kb) -> A_ {
      A_ a{0, 0, 0, 0};
      const int k = kb + lane;
      if (k < n_units) {
        const int64_t u = u0 + k;
        const int b = find_seq(P, p.B, u);
        const int np = (P[b + 1] - P[b]) / p.Hkv;
        const int rem = (int)(u - P[b]);
        const int h = rem / np, j = rem - h * np;
        a.h = h;
        a.pid = p.block_table[(int64_t)b * p.max_pages + j];
        const int ctx = p.ctx_lens[b];
        a.ntok = min(kPage, ctx - j * kPage);
        a.ok = 1;
      }
      return a;
    };
    auto phaseB = [&](const A_ &a) -> B_ {
      B_ r{0, 0, 0xffffu};
      if (a.ok && a.pid >= 0 && a.pid < p.num_pages) {
        if constexpr (ADA) {
          const spkv_page_hdr hd = p.hdr[a.pid];
          r.off16 = hd.code_off16;
          r.bits = hd.bits;
        }
        if (p.keep) r.keep = p.keep[(int64_t)a.pid * p.Hkv + a.h];
      }
      return r;
    };
    A_ an = phaseA(0);
    B_ bn = phaseB(an);
    int issued_round[Ly::NST];
#pragma unroll
    for (int s = 0; s < Ly::NST; ++s) issued_round[s] = -1;
    for (int kb = 0; kb < n_units; kb += 32) {
      const A_ ac = an;
      const B_ bc = bn;
      // finalise this lane's unit
      int valid = 0;
      uint64_t rec_off = 0, v_off = 0;
      uint32_t rec_sz = 0;
      if (ac.ok) {
        if (ac.pid < 0 || ac.pid >= p.num_pages) {
          set_err(p.err, SPKV_DEVERR_PAGE_ID);
        } else if (ADA && tier_of_bits(bc.bits) < 0) {
          set_err(p.err, SPKV_DEVERR_BITS);
        } else {
          v_off = ((uint64_t)ac.pid * p.Hkv + ac.h) * (kPage * kD);
          if constexpr (ADA) {
            rec_sz = rec_bytes(bc.bits);
            rec_off = (uint64_t)bc.off16 * 16u + (uint64_t)ac.h * rec_sz;
            if (rec_off + rec_sz > p.arena_bytes) set_err(p.err, SPKV_DEVERR_RECORD);
            else valid = 1;
          } else {
            valid = 1;
          }
        }
      }
      const uint32_t live = bc.keep & ((1u << ac.ntok) - 1u);
      an = phaseA(kb + 32);
      const int cnt = min(32, n_units - kb);
      for (int i = 0; i < cnt; ++i) {
        if (i == 16) bn = phaseB(an);
        const int k = kb + i;
        const int s = k % Ly::NST, r = k / Ly::NST;
        if (r > 0) mbar_wait_bounded(&empty[s], (uint32_t)(r - 1) & 1u, abort_flag, p.err);
        if (lane == i) {
          StageMeta m;
          m.valid = valid && !*abort_flag;
          m.bits = bc.bits;
          m.ntok = ac.ntok;
          m.live = live;
          meta[s] = m;
          uint8_t *st = stages + s * Ly::STAGE;
          if (m.valid) {
            if constexpr (ADA) {
              mbar_arrive_expect_tx(&full[s], rec_sz + 4096u);
              bulk_g2s(st, p.v_pages + v_off, 4096u, &full[s]);
              bulk_g2s(st + Ly::REC_OFF, p.arena + rec_off, rec_sz, &full[s]);
            } else {
              mbar_arrive_expect_tx(&full[s], 8192u);
              bulk_g2s(st, p.k_pages + v_off, 4096u, &full[s]);
              bulk_g2s(st + Ly::KV_OFF, p.v_pages + v_off, 4096u, &full[s]);
            }
          } else {
            mbar_arrive(&full[s]);
          }
        }
        issued_round[s] = r;
        __syncwarp();
      }
      if (cnt <= 16) bn = phaseB(an);
    }
    // On an abort, copies may still be in flight into our stages: wait for
    // them (bounded) before the CTA's shared memory can be released.
    if (*abort_flag && lane == 0) {
      volatile int dummy = 0;
      for (int s = 0; s < Ly::NST; ++s)
        if (issued_round[s] >= 0) mbar_wait_bounded(&full[s], (uint32_t)issued_round[s] & 1u, &dummy, nullptr);
    }
    return;
  }

  // ============================= consumer warps ============================
  const int ctid = tid;  // 0 .. 127
  float *pbuf = pbuf_all + wid * (kPage * G * 2);
  int64_t u = u0;
  int k = wid;  // next unit index of this warp (CTA-relative)
  while (u < u1) {
    const int b = find_seq(P, p.B, u);
    const int np = (P[b + 1] - P[b]) / p.Hkv;
    const int h = (int)((u - P[b]) / np);
    const int64_t seg_hi = (int64_t)P[b] + (int64_t)(h + 1) * np;
    const int64_t seg_end = seg_hi < u1 ? seg_hi : u1;
    const int bh = b * p.Hkv + h;

    // ---- per-segment query preparation
    for (int g = wid; g < G; g += kNCW) {
      const uint16_t *qrow = p.q + ((int64_t)b * p.Hq + (int64_t)h * G + g) * kD;
      if constexpr (ADA) {
        const float qn = ada_qprep_row<G, Ly::QT_HALF>(qrow, g, lpol, laz, uni, lane);
        if (lane == 0) sc[g] = qn * kLog2e * 0.08838834764831845f;
      } else {
        dense_qprep_row<G, Ly::QT_HALF>(qrow, g, uni, lane);
      }
    }
    if constexpr (ADA) {
      if (ctid == 0) {
        sc[G] = p.rad_lo[h];
        sc[G + 1] = p.rad_step[h];
      }
    }
    named_bar_sync(1, kNCW * 32);

    float m[G], lsum[G];
    float2 acc[G][2];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = kNegInf;
      lsum[g] = 0.f;
      acc[g][0] = acc[g][1] = make_float2(0.f, 0.f);
    }
    float scg[G];
#pragma unroll
    for (int g = 0; g < G; ++g) scg[g] = sc[g];
    const float Lh = ADA ? sc[G] : 0.f, Dh = ADA ? sc[G + 1] : 0.f;

    for (; u0 + k < seg_end; k += kNCW) {
      const int s = k % Ly::NST, r = k / Ly::NST;
      const bool ok = mbar_wait_bounded(&full[s], (uint32_t)r & 1u, abort_flag, p.err);
      const StageMeta mt = meta[s];
      const uint8_t *st = stages + s * Ly::STAGE;
      if (ok && mt.valid && mt.live) {
        float l2[G];
        if constexpr (ADA) {
          float f[G];
          const int ti = tier_of_bits(mt.bits);
          const float *qt = uni + ti * Ly::QT_TIER;
          const float2 *lp = lpol + lut_off(ti), *la = laz + lut_off(ti);
          const uint8_t *rec = st + Ly::REC_OFF;
          switch (mt.bits) {
            case 3: ada_page_f<3, G, Ly::QT_HALF>(rec, qt, lp, la, lane, f); break;
            case 4: ada_page_f<4, G, Ly::QT_HALF>(rec, qt, lp, la, lane, f); break;
            case 6: ada_page_f<6, G, Ly::QT_HALF>(rec, qt, lp, la, lane, f); break;
            default: ada_page_f<8, G, Ly::QT_HALF>(rec, qt, lp, la, lane, f); break;
          }
          const float rc = (float)rec[256 * mt.bits + (lane & 15)];
          const float rad = fast_exp2(fmaf(rc, Dh, Lh));
#pragma unroll
          for (int g = 0; g < G; ++g) l2[g] = scg[g] * rad * f[g];
        } else {
          dense_page_logits<G, Ly::QT_HALF>(st, uni, lane, l2);
        }
        const bool alive = lane < 16 && ((mt.live >> (lane & 15)) & 1u);
        float pg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float x = alive ? l2[g] : kNegInf;
          float mx = x;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float mnew = fmaxf(m[g], mx);
          const float alpha = mnew == kNegInf ? 1.f : fast_exp2(m[g] - mnew);
          pg[g] = alive ? fast_exp2(x - mnew) : 0.f;
          lsum[g] = fmaf(lsum[g], alpha, pg[g]);
          const float2 a2 = make_float2(alpha, alpha);
          acc[g][0] = fmul2(acc[g][0], a2);
          acc[g][1] = fmul2(acc[g][1], a2);
          m[g] = mnew;
        }
        if (lane < 16) {
          float *dst = pbuf + lane * G * 2;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            dst[2 * g] = pg[g];
            dst[2 * g + 1] = pg[g];
          }
        }
        __syncwarp();
        const uint8_t *vpage = ADA ? st : st + Ly::KV_OFF;
#pragma unroll
        for (int t = 0; t < kPage; ++t) {
          if ((mt.live >> t) & 1u) {
            const uint2 vw = *reinterpret_cast<const uint2 *>(vpage + t * 256 + lane * 8);
            const float2 v01 = make_float2(bf16lo(vw.x), bf16hi(vw.x));
            const float2 v23 = make_float2(bf16lo(vw.y), bf16hi(vw.y));
            const float *pp = pbuf + t * G * 2;
            if constexpr (G == 1) {
              const float2 p2 = *reinterpret_cast<const float2 *>(pp);
              acc[0][0] = ffma2(p2, v01, acc[0][0]);
              acc[0][1] = ffma2(p2, v23, acc[0][1]);
            } else {
#pragma unroll
              for (int g = 0; g < G; g += 2) {
                const float4 p4 = *reinterpret_cast<const float4 *>(pp + 2 * g);
                const float2 pa = make_float2(p4.x, p4.y), pb = make_float2(p4.z, p4.w);
                acc[g][0] = ffma2(pa, v01, acc[g][0]);
                acc[g][1] = ffma2(pa, v23, acc[g][1]);
                acc[g + 1][0] = ffma2(pb, v01, acc[g + 1][0]);
                acc[g + 1][1] = ffma2(pb, v23, acc[g + 1][1]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- merge the 4 warps' states of this segment into one partial
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], o);
    }
    named_bar_sync(1, kNCW * 32);  // every warp is done with the query table
    float *cmb = uni + wid * G * Ly::CMB;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float *cg = cmb + g * Ly::CMB;
      if (lane == 0) {
        cg[0] = m[g];
        cg[1] = lsum[g];
      }
      *reinterpret_cast<float4 *>(cg + 4 + 4 * lane) = make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
    }
    named_bar_sync(1, kNCW * 32);
    float *slot = p.ws + (int64_t)(c + bh) * G * Ly::CMB;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mw[kNCW], M = kNegInf;
#pragma unroll
      for (int w = 0; w < kNCW; ++w) {
        mw[w] = uni[(w * G + g) * Ly::CMB];
        M = fmaxf(M, mw[w]);
      }
      float num = 0.f, den = 0.f;
#pragma unroll
      for (int w = 0; w < kNCW; ++w) {
        const float s = mw[w] == kNegInf ? 0.f : fast_exp2(mw[w] - M);
        num = fmaf(s, uni[(w * G + g) * Ly::CMB + 4 + ctid], num);
        den = fmaf(s, uni[(w * G + g) * Ly::CMB + 1], den);
      }
      slot[g * Ly::CMB + 4 + ctid] = num;
      if (ctid == 0) {
        slot[g * Ly::CMB + 0] = M;
        slot[g * Ly::CMB + 1] = den;
      }
    }
    named_bar_sync(1, kNCW * 32);  // the union region is reused by the next query table
    u = seg_end;
  }
}

// ------------------------------------------------------------ merge kernel
// One block per (sequence, kv head): combine the partials of the splits that
// covered its units, for its G query heads.  out = sum_s 2^(m_s - M) acc_s /
// sum_s 2^(m_s - M) l_s, or 0 when no slot was retained.
template <int G>
__global__ void __launch_bounds__(128) merge_kernel(const float *ws, int C, const int32_t *ctx_lens, int B, int Hkv,
                                                    int Hq, int max_ctx, int max_pages, void *out, int out_bf16) {
  constexpr int CMB = 132;
  __shared__ int64_t red[2][4];
  const int bh = blockIdx.x, b = bh / Hkv, h = bh % Hkv;
  const int tid = threadIdx.x;
  int64_t before = 0, total = 0;
  for (int i = tid; i < B; i += 128) {
    const int np = seq_pages(ctx_lens[i], max_ctx, max_pages, nullptr) * Hkv;
    total += np;
    if (i < b) before += np;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  if ((tid & 31) == 0) {
    red[0][tid >> 5] = before;
    red[1][tid >> 5] = total;
  }
  __syncthreads();
  before = red[0][0] + red[0][1] + red[0][2] + red[0][3];
  const int64_t W = red[1][0] + red[1][1] + red[1][2] + red[1][3];
  const int np = seq_pages(ctx_lens[b], max_ctx, max_pages, nullptr);
  const int64_t a = before + (int64_t)h * np, e = a + np;
  float res[G];
#pragma unroll
  for (int g = 0; g < G; ++g) res[g] = 0.f;
  if (np > 0) {
    const int64_t cf = ((a + 1) * C + W - 1) / W - 1;
    int64_t cl = (e * C + W - 1) / W - 1;
    if (cl > C - 1) cl = C - 1;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float M = kNegInf;
      for (int64_t cc = cf; cc <= cl; ++cc) {
        if (split_begin(W, C, (int)cc) >= split_begin(W, C, (int)cc + 1)) continue;
        M = fmaxf(M, ws[((cc + bh) * G + g) * CMB]);
      }
      float num = 0.f, den = 0.f;
      if (M != kNegInf) {
        for (int64_t cc = cf; cc <= cl; ++cc) {
          if (split_begin(W, C, (int)cc) >= split_begin(W, C, (int)cc + 1)) continue;
          const float *sl = ws + ((cc + bh) * G + g) * CMB;
          const float mm = sl[0];
          const float s = mm == kNegInf ? 0.f : fast_exp2(mm - M);
          num = fmaf(s, sl[4 + tid], num);
          den = fmaf(s, sl[1], den);
        }
      }
      res[g] = den > 0.f ? num / den : 0.f;
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int64_t o = ((int64_t)b * Hq + (int64_t)h * G + g) * kD + tid;
    if (out_bf16) reinterpret_cast<__nv_bfloat16 *>(out)[o] = __float2bfloat16_rn(res[g]);
    else reinterpret_cast<float *>(out)[o] = res[g];
  }
}

// ---------------------------------------------------- decompress kernel
// k~ = bf16(r~ u~(c)) for one (page, kv head) per block of 32 threads; the
// strawman path of the summary's problem statement (writes dense keys to HBM).
__global__ void __launch_bounds__(32) decompress_kernel(SplitParams p, uint16_t *kout) {
  __shared__ float2 lpol[kLutEntries], laz[kLutEntries];
  __shared__ __align__(16) uint8_t rec[2064];
  __shared__ __align__(16) uint16_t tile[kPage * kD];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z, lane = threadIdx.x;
  const int np = seq_pages(p.ctx_lens[b], p.max_ctx, p.max_pages, nullptr);
  if (j >= np) return;
  const int pid = p.block_table[(int64_t)b * p.max_pages + j];
  if (pid < 0 || pid >= p.num_pages) {
    if (lane == 0) set_err(p.err, SPKV_DEVERR_PAGE_ID);
    return;
  }
  const spkv_page_hdr hd = p.hdr[pid];
  const int ti = tier_of_bits(hd.bits);
  if (ti < 0) {
    if (lane == 0) set_err(p.err, SPKV_DEVERR_BITS);
    return;
  }
  const uint32_t rsz = rec_bytes(hd.bits);
  const uint64_t roff = (uint64_t)hd.code_off16 * 16u + (uint64_t)h * rsz;
  if (roff + rsz > p.arena_bytes) {
    if (lane == 0) set_err(p.err, SPKV_DEVERR_RECORD);
    return;
  }
  build_luts(lpol, laz, lane, 32);
  for (uint32_t i = lane * 16; i < rsz; i += 32 * 16)
    *reinterpret_cast<uint4 *>(rec + i) = *reinterpret_cast<const uint4 *>(p.arena + roff + i);
  __syncwarp();
  const int t = lane & 15, half = lane >> 4;
  const float2 *lp = lpol + lut_off(ti), *la = laz + lut_off(ti);
  const float Lh = p.rad_lo[h], Dh = p.rad_step[h];
  const float rad = exp2f(fmaf((float)rec[256 * hd.bits + t], Dh, Lh));
  // decode this lane's 64 components with the same prefix chain as ADA, then
  // scale the second half by the first half's sine product
  float u[64];
  float Pp = 1.0f;
  auto run = [&](auto bits_tag) {
    constexpr int BITS = decltype(bits_tag)::value;
    uint32_t W[2 * BITS];
    const uint32_t *rw = reinterpret_cast<const uint32_t *>(rec);
    // gather the slot's 2b words of this half from the chunk-major layout
#pragma unroll
    for (int w = 0; w < 2 * BITS; ++w) {
      const int gw = half * 2 * BITS + w;  // global word index in the slot's stream
      W[w] = rw[((gw >> 2) * 16 + t) * 4 + (gw & 3)];
    }
#pragma unroll
    for (int a = 0; a < 64; ++a) {
      const uint32_t cc = code_at<BITS>(W, a);
      float2 e;
      if (a == 62 && half) e = la[cc];
      else if (a == 63 && half) e = make_float2(1.0f, 0.0f);
      else e = lp[cc];
      u[a] = Pp * e.x;
      Pp *= e.y;
    }
  };
  switch (hd.bits) {
    case 3: run(std::integral_constant<int, 3>{}); break;
    case 4: run(std::integral_constant<int, 4>{}); break;
    case 6: run(std::integral_constant<int, 6>{}); break;
    default: run(std::integral_constant<int, 8>{}); break;
  }
  const float P64 = __shfl_sync(0xffffffffu, Pp, t);  // first-half product of slot t
  const float scale = half ? rad * P64 : rad;
#pragma unroll
  for (int a = 0; a < 64; ++a) tile[t * kD + half * 64 + a] = __bfloat16_as_ushort(__float2bfloat16_rn(scale * u[a]));
  __syncwarp();
  uint16_t *dst = kout + ((int64_t)pid * p.Hkv + h) * (kPage * kD);
  for (int i = lane; i < kPage * kD / 8; i += 32)
    reinterpret_cast<uint4 *>(dst)[i] = reinterpret_cast<const uint4 *>(tile)[i];
}

// ------------------------------------------------------ debug logits
// logits[b, hq, 16 j + t] = ||q|| r~ f_b / sqrt(d) for one page per block
// (one warp); same query coding and f_b device code as the split kernel.
template <int G>
__global__ void __launch_bounds__(32) debug_logits_kernel(SplitParams p, float *logits) {
  constexpr int QT_HALF = 64 * G + 4;
  __shared__ float2 lpol[kLutEntries], laz[kLutEntries];
  __shared__ __align__(16) float qt[kTiers * 2 * QT_HALF];
  __shared__ __align__(16) uint8_t rec[2064];
  __shared__ float qn[G];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z, lane = threadIdx.x;
  const int ctx = p.ctx_lens[b];
  const int np = seq_pages(ctx, p.max_ctx, p.max_pages, p.err);
  if (j >= np) return;
  const int pid = p.block_table[(int64_t)b * p.max_pages + j];
  if (pid < 0 || pid >= p.num_pages) {
    if (lane == 0) set_err(p.err, SPKV_DEVERR_PAGE_ID);
    return;
  }
  const spkv_page_hdr hd = p.hdr[pid];
  const int ti = tier_of_bits(hd.bits);
  if (ti < 0) {
    if (lane == 0) set_err(p.err, SPKV_DEVERR_BITS);
    return;
  }
  const uint32_t rsz = rec_bytes(hd.bits);
  const uint64_t roff = (uint64_t)hd.code_off16 * 16u + (uint64_t)h * rsz;
  if (roff + rsz > p.arena_bytes) {
    if (lane == 0) set_err(p.err, SPKV_DEVERR_RECORD);
    return;
  }
  build_luts(lpol, laz, lane, 32);
  for (uint32_t i = lane * 16; i < rsz; i += 32 * 16)
    *reinterpret_cast<uint4 *>(rec + i) = *reinterpret_cast<const uint4 *>(p.arena + roff + i);
  __syncwarp();
  for (int g = 0; g < G; ++g) {
    const float n = ada_qprep_row<G, QT_HALF>(p.q + ((int64_t)b * p.Hq + (int64_t)h * G + g) * kD, g, lpol, laz,
                                              qt, lane);
    if (lane == 0) qn[g] = n;
  }
  __syncwarp();
  float f[G];
  const float *q0 = qt + ti * 2 * QT_HALF;
  const float2 *lp = lpol + lut_off(ti), *la = laz + lut_off(ti);
  switch (hd.bits) {
    case 3: ada_page_f<3, G, QT_HALF>(rec, q0, lp, la, lane, f); break;
    case 4: ada_page_f<4, G, QT_HALF>(rec, q0, lp, la, lane, f); break;
    case 6: ada_page_f<6, G, QT_HALF>(rec, q0, lp, la, lane, f); break;
    default: ada_page_f<8, G, QT_HALF>(rec, q0, lp, la, lane, f); break;
  }
  const int t = lane;
  if (t < 16 && j * kPage + t < ctx) {
    const float rad = exp2f(fmaf((float)rec[256 * hd.bits + t], p.rad_step[h], p.rad_lo[h]));
    const uint32_t keep = p.keep ? p.keep[(int64_t)pid * p.Hkv + h] : 0xffffu;
    for (int g = 0; g < G; ++g) {
      const float v = ((keep >> t) & 1u) ? qn[g] * rad * f[g] * 0.08838834764831845f : kNegInf;
      logits[((int64_t)b * p.Hq + (int64_t)h * G + g) * p.max_ctx + j * kPage + t] = v;
    }
  }
}

// ------------------------------------------------------------- host side
// Opt the kernel into the largest dynamic shared memory it can ask for (once
// per device) and report how many CTAs of `smem` bytes fit on one SM.
template <bool ADA, int G>
int blocks_per_sm(size_t smem) {
  static int configured[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(split_kernel<ADA, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Layout<ADA, G>::bytes(kMaxB)) != cudaSuccess)
      return -1;
    configured[dev] = 1;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, split_kernel<ADA, G>, kThreads, smem) != cudaSuccess)
    return -1;
  return n;
}

template <bool ADA>
int blocks_per_sm_for(int G, size_t smem) {
  switch (G) {
    case 1: return blocks_per_sm<ADA, 1>(smem);
    case 2: return blocks_per_sm<ADA, 2>(smem);
    case 4: return blocks_per_sm<ADA, 4>(smem);
    case 8: return blocks_per_sm<ADA, 8>(smem);
  }
  return -1;
}

template <bool ADA>
size_t smem_for(int G, int B) {
  switch (G) {
    case 1: return Layout<ADA, 1>::bytes(B);
    case 2: return Layout<ADA, 2>::bytes(B);
    case 4: return Layout<ADA, 4>::bytes(B);
    case 8: return Layout<ADA, 8>::bytes(B);
  }
  return 0;
}

bool g_supported(int G) { return G == 1 || G == 2 || G == 4 || G == 8; }

// Default split count: every resident CTA slot of the device, but at most one
// split per 8 units of the largest batch these sizes allow.
int default_splits(int B, int Hkv, int max_ctx) {
  const int sms = device_sm_count();
  if (sms <= 0) return -1;
  const int64_t units = (int64_t)B * Hkv * ((max_ctx + kPage - 1) / kPage);
  int64_t c = (int64_t)sms * 2;
  if (units / 8 < c) c = units / 8;
  if (c < 1) c = 1;
  return (int)c;
}

struct DecodeArgs {
  SplitParams sp;
  int G, num_splits;
  void *out;
  int out_bf16;
};

template <bool ADA>
spkv_status launch_split_and_merge(const DecodeArgs &a, cudaStream_t stream) {
  const size_t smem = smem_for<ADA>(a.G, a.sp.B);
  if (blocks_per_sm_for<ADA>(a.G, smem) < 1) return SPKV_ERR_CUDA;
  const int C = a.num_splits;
  switch (a.G) {
    case 1: split_kernel<ADA, 1><<<C, kThreads, smem, stream>>>(a.sp); break;
    case 2: split_kernel<ADA, 2><<<C, kThreads, smem, stream>>>(a.sp); break;
    case 4: split_kernel<ADA, 4><<<C, kThreads, smem, stream>>>(a.sp); break;
    case 8: split_kernel<ADA, 8><<<C, kThreads, smem, stream>>>(a.sp); break;
  }
  if (cudaGetLastError() != cudaSuccess) return SPKV_ERR_CUDA;
  const int nb = a.sp.B * a.sp.Hkv;
  switch (a.G) {
    case 1: merge_kernel<1><<<nb, 128, 0, stream>>>(a.sp.ws, C, a.sp.ctx_lens, a.sp.B, a.sp.Hkv, a.sp.Hq, a.sp.max_ctx, a.sp.max_pages, a.out, a.out_bf16); break;
    case 2: merge_kernel<2><<<nb, 128, 0, stream>>>(a.sp.ws, C, a.sp.ctx_lens, a.sp.B, a.sp.Hkv, a.sp.Hq, a.sp.max_ctx, a.sp.max_pages, a.out, a.out_bf16); break;
    case 4: merge_kernel<4><<<nb, 128, 0, stream>>>(a.sp.ws, C, a.sp.ctx_lens, a.sp.B, a.sp.Hkv, a.sp.Hq, a.sp.max_ctx, a.sp.max_pages, a.out, a.out_bf16); break;
    case 8: merge_kernel<8><<<nb, 128, 0, stream>>>(a.sp.ws, C, a.sp.ctx_lens, a.sp.B, a.sp.Hkv, a.sp.Hq, a.sp.max_ctx, a.sp.max_pages, a.out, a.out_bf16); break;
  }
  return cudaGetLastError() == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}

size_t ws_bytes_for(int B, int Hq, int Hkv, int C) {
  return (size_t)(C + B * Hkv) * (size_t)(Hq / Hkv) * 132u * sizeof(float);
}

// Shared validation of the batch arguments; fills sp's batch fields.
spkv_status prep_batch(SplitParams &sp, int Hkv, const uint16_t *q, int B, int Hq, const int32_t *block_table,
                       int max_pages, const int32_t *ctx_lens, int max_ctx, void *out, void *ws, size_t ws_bytes,
                       int num_splits, int *G_out, int *C_out) {
  if (B < 0 || Hq < 1 || max_pages < 0 || max_ctx < 0 || num_splits < 0) return SPKV_ERR_INVALID_ARG;
  if (Hq % Hkv) return SPKV_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (!g_supported(G)) return SPKV_ERR_UNSUPPORTED;
  if (B > kMaxB) return SPKV_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv * ((int64_t)max_ctx + kPage - 1) / kPage > (int64_t)1 << 30) return SPKV_ERR_UNSUPPORTED;
  if (B > 0 && (!q || !block_table || !ctx_lens || !out)) return SPKV_ERR_INVALID_ARG;
  if (((uintptr_t)q & 7) || ((uintptr_t)ws & 15) || ((uintptr_t)out & 15)) return SPKV_ERR_INVALID_ARG;
  int C = num_splits ? num_splits : default_splits(B, Hkv, max_ctx);
  if (C < 1) return SPKV_ERR_CUDA;
  if (ws_bytes < ws_bytes_for(B, Hq, Hkv, C) || (B > 0 && !ws)) return SPKV_ERR_WORKSPACE;
  sp.q = q;
  sp.B = B;
  sp.Hq = Hq;
  sp.block_table = block_table;
  sp.max_pages = max_pages;
  sp.ctx_lens = ctx_lens;
  sp.max_ctx = max_ctx;
  sp.ws = reinterpret_cast<float *>(ws);
  *G_out = G;
  *C_out = C;
  return SPKV_OK;
}

void fill_cache(SplitParams &sp, const spkv_cache *c) {
  sp.arena = c->code_arena;
  sp.arena_bytes = c->code_arena_bytes;
  sp.hdr = c->hdr;
  sp.rad_lo = c->rad_lo_log2;
  sp.rad_step = c->rad_step_log2;
  sp.k_pages = nullptr;
  sp.v_pages = c->v_pages;
  sp.keep = c->keep_mask;
  sp.err = c->err_flags;
  sp.Hkv = c->num_kv_heads;
  sp.num_pages = c->num_pages;
}

}  // namespace
}  // namespace spkv

using namespace spkv;

extern "C" int32_t spkv_decode_default_splits(int32_t B, int32_t num_kv_heads, int32_t max_ctx) {
  if (B < 0 || num_kv_heads < 1 || max_ctx < 0) return -1;
  return default_splits(B, num_kv_heads, max_ctx);
}

extern "C" size_t spkv_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t max_ctx,
                                              int32_t num_splits) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || max_ctx < 0 || num_splits < 0) return 0;
  const int C = num_splits ? num_splits : default_splits(B, Hkv, max_ctx);
  if (C < 1) return 0;
  return ws_bytes_for(B, Hq, Hkv, C);
}

extern "C" spkv_status spkv_decode_attention(const spkv_cache *cache, const uint16_t *q, int32_t B, int32_t Hq,
                                             const int32_t *block_table, int32_t max_pages,
                                             const int32_t *ctx_lens, int32_t max_ctx, void *out,
                                             int32_t out_is_bf16, void *ws, size_t ws_bytes, int32_t num_splits,
                                             void *stream) {
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  DecodeArgs a;
  fill_cache(a.sp, cache);
  st = prep_batch(a.sp, cache->num_kv_heads, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, out, ws, ws_bytes,
                  num_splits, &a.G, &a.num_splits);
  if (st != SPKV_OK) return st;
  if (B == 0) return SPKV_OK;
  a.out = out;
  a.out_bf16 = out_is_bf16 ? 1 : 0;
  return launch_split_and_merge<true>(a, (cudaStream_t)stream);
}

extern "C" spkv_status spkv_dense_decode(const uint16_t *k_pages, const uint16_t *v_pages, int32_t num_pages,
                                         int32_t Hkv, const uint16_t *keep_mask, uint32_t *err_flags,
                                         const uint16_t *q, int32_t B, int32_t Hq, const int32_t *block_table,
                                         int32_t max_pages, const int32_t *ctx_lens, int32_t max_ctx, void *out,
                                         int32_t out_is_bf16, void *ws, size_t ws_bytes, int32_t num_splits,
                                         void *stream) {
  if (!k_pages || !v_pages || num_pages < 0 || Hkv < 1) return SPKV_ERR_INVALID_ARG;
  if (((uintptr_t)k_pages & 15) || ((uintptr_t)v_pages & 15)) return SPKV_ERR_INVALID_ARG;
  DecodeArgs a;
  a.sp = SplitParams{};
  a.sp.k_pages = k_pages;
  a.sp.v_pages = v_pages;
  a.sp.keep = keep_mask;
  a.sp.err = err_flags;
  a.sp.Hkv = Hkv;
  a.sp.num_pages = num_pages;
  spkv_status st = prep_batch(a.sp, Hkv, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, out, ws, ws_bytes,
                              num_splits, &a.G, &a.num_splits);
  if (st != SPKV_OK) return st;
  if (B == 0) return SPKV_OK;
  a.out = out;
  a.out_bf16 = out_is_bf16 ? 1 : 0;
  return launch_split_and_merge<false>(a, (cudaStream_t)stream);
}

extern "C" spkv_status spkv_decompress_then_dot(const spkv_cache *cache, uint16_t *k_scratch, const uint16_t *q,
                                                int32_t B, int32_t Hq, const int32_t *block_table,
                                                int32_t max_pages, const int32_t *ctx_lens, int32_t max_ctx,
                                                void *out, int32_t out_is_bf16, void *ws, size_t ws_bytes,
                                                int32_t num_splits, void *stream) {
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  if (!k_scratch || ((uintptr_t)k_scratch & 15)) return SPKV_ERR_INVALID_ARG;
  DecodeArgs a;
  fill_cache(a.sp, cache);
  st = prep_batch(a.sp, cache->num_kv_heads, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, out, ws, ws_bytes,
                  num_splits, &a.G, &a.num_splits);
  if (st != SPKV_OK) return st;
  if (B == 0 || max_pages == 0) return SPKV_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int pages_used = std::min(max_pages, (max_ctx + kPage - 1) / kPage);
  if (pages_used > 0) {
    dim3 grid(pages_used, cache->num_kv_heads, B);
    decompress_kernel<<<grid, 32, 0, s>>>(a.sp, k_scratch);
    if (cudaGetLastError() != cudaSuccess) return SPKV_ERR_CUDA;
  }
  a.sp.k_pages = k_scratch;
  a.out = out;
  a.out_bf16 = out_is_bf16 ? 1 : 0;
  return launch_split_and_merge<false>(a, s);
}

extern "C" spkv_status spkv_debug_logits(const spkv_cache *cache, const uint16_t *q, int32_t B, int32_t Hq,
                                         const int32_t *block_table, int32_t max_pages, const int32_t *ctx_lens,
                                         int32_t max_ctx, float *logits, void *stream) {
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  if (B < 0 || Hq < 1 || max_pages < 0 || max_ctx < 0 || Hq % cache->num_kv_heads) return SPKV_ERR_INVALID_ARG;
  const int G = Hq / cache->num_kv_heads;
  if (!g_supported(G)) return SPKV_ERR_UNSUPPORTED;
  if (B == 0 || max_ctx == 0) return SPKV_OK;
  if (!q || !block_table || !ctx_lens || !logits || ((uintptr_t)q & 7)) return SPKV_ERR_INVALID_ARG;
  SplitParams sp;
  fill_cache(sp, cache);
  sp.q = q;
  sp.B = B;
  sp.Hq = Hq;
  sp.block_table = block_table;
  sp.max_pages = max_pages;
  sp.ctx_lens = ctx_lens;
  sp.max_ctx = max_ctx;
  sp.ws = nullptr;
  const int pages_used = std::min(max_pages, (max_ctx + kPage - 1) / kPage);
  if (pages_used == 0) return SPKV_OK;
  dim3 grid(pages_used, cache->num_kv_heads, B);
  cudaStream_t s = (cudaStream_t)stream;
  switch (G) {
    case 1: debug_logits_kernel<1><<<grid, 32, 0, s>>>(sp, logits); break;
    case 2: debug_logits_kernel<2><<<grid, 32, 0, s>>>(sp, logits); break;
    case 4: debug_logits_kernel<4><<<grid, 32, 0, s>>>(sp, logits); break;
    case 8: debug_logits_kernel<8><<<grid, 32, 0, s>>>(sp, logits); break;
  }
  return cudaGetLastError() == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}
