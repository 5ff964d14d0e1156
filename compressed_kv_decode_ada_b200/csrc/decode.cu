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
//    sequence-major; split c of C owns a contiguous range cut at equal steps
//    of a weighted position (every kv-row boundary costs a few units: see
//    Partition), so C = 2 x SMs CTAs is one balanced wave.
//  * CTA = 1 producer warp + 5 consumer warps (4 for G = 8), 2 CTAs per SM.
//    The producer resolves block table -> page header -> record address and
//    streams each unit's code record (256 b + 16 bytes) into a shared-memory
//    ring with 1-D bulk copies (cp.async.bulk, mbarrier completion); with
//    several tiers it walks each segment tier by tier.  Consumer warp w takes
//    pairs of units w, w + NCW, ..., fetches the pair's value pages itself
//    (3-D TMA, 128-byte swizzle) and keeps its own online-softmax state.
//  * f_b: lane = (slot t, half of the angle chain) of both pages of a pair.
//    Each lane decodes 64 angle codes per page, looks up (cos, sin) of the
//    cell midpoint in a shared-memory table and runs the prefix product of
//    sines
//        u_j = (prod_{i<j} sin phi_i) cos phi_j,
//    accumulating <u_q, u_k> for the G query heads of the kv head on CUDA
//    cores (f32x2 FMAs).  The two halves are joined by
//        f = A + (prod_{i<=64} sin phi_i) * B.
//    The key's unit vector lives only in registers.
//  * Online softmax in the log2 domain with a lazily moving maximum; P.V on
//    tensor cores (mma.sync m16n8k16 bf16, P split into bf16 hi + lo).
//  * Per segment every consumer warp writes one partial (m, l, acc[128]) per
//    query head and counts it on its kv row; the merge kernel, launched as a
//    programmatic dependent, merges each row once its partials are counted.
#include <cuda_bf16.h>

#include <type_traits>

#include "spkv_encode.cuh"

namespace spkv {

spkv_status check_cache(const spkv_cache *c);
int device_sm_count();
bool make_value_tensor_map(CUtensorMap *map, const void *v_pages, uint64_t rows);

namespace {

constexpr int kNCWMax = 6;                   // largest consumer-warp count of any path
constexpr int kIssue = 8;                    // units the producer warp issues per step
constexpr float kRescaleSlack = 8.0f;        // log2 units a running max may lag the true max
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

// float2 load from a 32-bit shared-window address of a table that is
// written once before the consumer loop (so the load may move freely).
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// Tensor-core helpers for P.V: one m16n8k16 bf16 MMA with fp32 accumulation,
// and a transposing 4-tile ldmatrix.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}
// (x, y) -> bf16x2 (x in the low half), round to nearest, and the bf16x2 of
// the rounding residuals: x ~= hi + lo to about 16 significant bits.
__device__ __forceinline__ void split_bf16x2(float x, float y, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Warp-wide max of a float through an order-preserving integer key and one
// redux.sync (NaN-free inputs; -inf allowed).
__device__ __forceinline__ float warp_max(float x) {
  const int i = __float_as_int(x);
  const int key = i >= 0 ? i : (i ^ 0x7fffffff);
  const int r = __reduce_max_sync(0xffffffffu, key);
  return __int_as_float(r >= 0 ? r : (r ^ 0x7fffffff));
}

// ----------------------------------------------------------------- layout
template <bool ADA, int G, bool NW = false>
struct Layout {
  // NCW consumer warps take PAIRS of units (ADA: the two pages of a pair that
  // share a tier share every query load).  The producer warp streams
  // only the small per-unit data -- the code record (ADA) or the bf16 K page
  // (dense) -- through a CTA-wide ring of NST stages; each consumer warp
  // fetches the value pages of its pair itself, into two private slots, when
  // it starts the pair, so the V loads overlap the logit computation and a
  // ring stage is released as soon as the logits are done.
  static constexpr int NCW = G <= 4 ? 5 : 4;
  static constexpr int THREADS = (NCW + 1) * 32;               // + producer warp
  // NW ("narrow", ADA only): every page has b <= 4, so a stage holds at most
  // a 1040-byte record and the ring has twice the stages in the same bytes.
  static constexpr int NST = ADA ? (NW ? (G == 8 ? 32 : 40) : (G == 8 ? 16 : 20)) : (G <= 4 ? 10 : 16);
  static_assert(NST >= kIssue, "one producer step must touch distinct stages");
  // Pair i uses stages 2i, 2i + 1 (mod NST) and belongs to warp i % NCW, so
  // with NST / 2 a multiple of NCW every use of a stage is by one warp, in
  // order: its parity waits always target the current or the next phase.
  static_assert((NST / 2) % NCW == 0, "a stage must belong to one consumer warp");
  // A value page lands through one 3-D TMA box (64 dims x 16 rows x 2 halves,
  // 128-byte swizzle): half j (dims 64 j .. 64 j + 63) at +2048 j, row t's
  // 16-byte chunk c at chunk c ^ (t & 7), so the transposing ldmatrix reads
  // of 8 consecutive rows hit 8 distinct bank groups.  1024-byte aligned.
  static constexpr int VSLOT = 4096;
  static constexpr int XSTAGE = ADA ? (NW ? 1040 : 2064) : 4096;  // code record | dense K page
  static constexpr int QT_HALF = ADA ? (64 * G + 4) : 8 * (8 * G + 4);  // floats, +16 B skew
  static constexpr int QT_TIER = 2 * QT_HALF;
  static constexpr int QT_FLOATS = (ADA ? kTiers : 1) * QT_TIER;
  static constexpr int PBUF_FLOATS = NCW * G * 2 * kPage;      // p[g][32 slots of 2 pages] per warp
  static constexpr int PB_BYTES = PBUF_FLOATS * 4;
  static constexpr int off_v = 0;                                 // NCW x 2 value slots
  static constexpr int off_x = off_v + NCW * 2 * VSLOT;           // ring stages
  // float2 single-angle tables: polar at off_lut, azimuth 384 entries later;
  // off_lut = 192 (mod 256) puts both b = 4 tables (entry 8 on) on 256-byte
  // boundaries: one 128-byte row each, and an entry's address is the
  // table's upper bytes with the entry offset as the low byte
  static constexpr int off_lut = (off_x + NST * XSTAGE + 255) / 256 * 256 + 192;
  static constexpr int LAZ_OFF = 384;  // entries
  static constexpr int lut_bytes = ADA ? (LAZ_OFF + kLutEntries) * 8 : 0;
  static constexpr int off_qt = off_lut + lut_bytes;
  static constexpr int off_pbuf = off_qt + QT_FLOATS * 4;
  static constexpr int off_sc = off_pbuf + PB_BYTES;            // G scales + L_h + Delta_h
  static constexpr int off_bar = off_sc + ((G + 2) * 4 + 15) / 16 * 16;  // full, empty, value slots
  static constexpr int off_meta = off_bar + (2 * NST + 2 * NCW) * 8;
  static constexpr int off_misc = off_meta + NST * 32;            // abort flag + scan scratch
  // the producer's own fp64 edge tables and code scratch (fused append)
  static constexpr int off_pe = (off_misc + 16 + 36 * 4 + 15) / 16 * 16;
  static constexpr int pe_bytes = ADA ? 2 * kLutEntries * 8 + 128 : 0;
  static constexpr int off_P = off_pe + pe_bytes;
  // + 1024 bytes of slack to align the carve-up base to 1024
  static constexpr size_t bytes(int B) { return (size_t)off_P + (size_t)(B + 1) * 4 + 16 + 1024; }
  // two CTAs per SM: 228 KB of shared memory minus 1 KB reserved per CTA
  static_assert(bytes(kMaxB) <= (228 * 1024 - 2 * 1024) / 2, "two CTAs per SM must fit");
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
  uint32_t tiers;  // tiers the query is coded for (bit t: b = {3,4,6,8}[t])
  uint32_t flags;  // SPKV_DECODE_* bits
  // fused single-token append (ADA only): the key and value [B, H_kv, 128] of
  // each sequence's token ctx - 1, encoded into its page before it is read;
  // nullptr: no append
  const uint16_t *new_k, *new_v;
  int Hkv, num_pages;
  const uint16_t *q;
  int B, Hq;
  const int32_t *block_table;
  int max_pages;
  const int32_t *ctx_lens;
  int max_ctx;
  float *ws;
  uint32_t *row_done;  // per kv row: consumer-warp partials written (zeroed before the launch)
};

// Stage metadata written by the producer, read by the consumer.
struct StageMeta {
  int valid;   // 0: skip this unit (bad page / header / record)
  int bits;    // ADA tier bit width
  int ntok;    // valid slots in the page (1..16)
  uint32_t live;  // keep-mask bits restricted to the first ntok slots
  int vrow;    // first row of the unit's value page in the value tensor map
  int pad[3];
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
// each tier's b with the same exact fp64 edge tests as the keys) -> decoded
// unit vector per tier, written to
// qt[tier * QT_TIER + half * QT_HALF + (pair * G + g) * 2 + e] for field
// a = 64 half + 2 pair + e.  Returns ||q||.
template <int G, int QT_HALF>
__device__ float ada_qprep_row(const uint16_t *qrow, int g, const float2 *lpol, const float2 *laz,
                               const double *pol_c2, const double *az_c2, float *qt, int lane, uint32_t tiers,
                               bool exact) {
  const uint2 raw = *reinterpret_cast<const uint2 *>(qrow + 4 * lane);
  double x[4], S[4];
  lane_suffix_sums(raw, lane, x, S);
  const double x127 = __shfl_sync(0xffffffffu, x[3], 31);
  const double qn = sqrt(__shfl_sync(0xffffffffu, S[0], 0));
#pragma unroll
  for (int ti = 0; ti < kTiers; ++ti) {
    if (!((tiers >> ti) & 1u)) continue;
    if (exact) {  // the exact-query variant: q / ||q|| itself, for every tier
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int a = 4 * lane + k;
        const int half = a >> 6, s = a & 63;
        qt[ti * 2 * QT_HALF + half * QT_HALF + ((s >> 1) * G + g) * 2 + (s & 1)] =
            qn > 0.0 ? (float)(x[k] / qn) : 0.0f;
      }
      continue;
    }
    int c[4];
    switch (ti) {
      case 0: lane_codes<3>(x, S, x127, lane, pol_c2, az_c2, c); break;
      case 1: lane_codes<4>(x, S, x127, lane, pol_c2, az_c2, c); break;
      case 2: lane_codes<6>(x, S, x127, lane, pol_c2, az_c2, c); break;
      default: lane_codes<8>(x, S, x127, lane, pol_c2, az_c2, c); break;
    }
    float2 cs[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int a = 4 * lane + k;
      if (a < 126) cs[k] = lpol[lut_off(ti) + c[k]];
      else if (a == 126) cs[k] = laz[lut_off(ti) + c[k]];
      else cs[k] = make_float2(1.0f, 0.0f);  // padding field: u_127 = product of all sines
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

// NB bits of a lane's code words starting at bit `bit` (compile-time after unrolling).
template <int NB, int NW>
__device__ __forceinline__ uint32_t bits_at(const uint32_t (&W)[NW], int bit) {
  const int w = bit >> 5, sh = bit & 31;
  uint32_t v;
  if (sh + NB <= 32) v = W[w] >> sh;
  else v = __funnelshift_r(W[w], W[w + 1], sh);
  return v & ((1u << NB) - 1u);
}
// 8 x (NB bits of the lane's code words starting at bit `bit`): the byte
// offset of the code's float2 table entry, one shift and one mask.
template <int NB, int NW>
__device__ __forceinline__ uint32_t off8_at(const uint32_t (&W)[NW], int bit) {
  const int w = bit >> 5, sh = bit & 31;
  constexpr uint32_t m = ((1u << NB) - 1u) << 3;
  if (sh + NB <= 32) return (sh >= 3 ? W[w] >> (sh - 3) : W[w] << (3 - sh)) & m;
  return __funnelshift_r(W[w], W[w + 1], sh - 3) & m;  // (sh > 32 - NB >= 24: sh - 3 >= 0)
}
template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&W)[2 * BITS], int a) {
  return bits_at<BITS, 2 * BITS>(W, a * BITS);
}

// f_b for the 16 slots of one record and the G heads (valid on lanes 0..15).
// Lane (t, half) runs the prefix product over the 64 fields of its half as two
// independent sub-chains of 32 fields (A = A1 + P1 A2), and the halves are
// joined with f = A_0 + P_0 A_1 (P_0 the product of the first half's sines).
// (cos, sin) of a field comes from the tier's 2^b-entry table; for b = 4 the
// 16 float2 entries fill one 128-byte row, so the gathers are conflict-free.
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
  const float2 *l62 = half ? laz : lpol;  // field 126 of the second half is the azimuth
  float2 acc[2][G];
  float Ps[2];
#pragma unroll
  for (int sc = 0; sc < 2; ++sc) {
    Ps[sc] = 1.f;
#pragma unroll
    for (int g = 0; g < G; ++g) acc[sc][g] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int pq = 0; pq < 16; ++pq) {
#pragma unroll
    for (int sc = 0; sc < 2; ++sc) {
      const int pp = pq + 16 * sc;  // pair index in this half: fields 2 pp, 2 pp + 1
      const uint32_t c0 = code_at<BITS>(W, 2 * pp), c1 = code_at<BITS>(W, 2 * pp + 1);
      float2 e0, e1;
      if (pp == 31) {
        e0 = l62[c0];
        const float2 t1 = lpol[half ? 0u : c1];
        e1 = make_float2(half ? 1.0f : t1.x, half ? 0.0f : t1.y);  // padding field: (1, 0)
      } else {
        e0 = lpol[c0];
        e1 = lpol[c1];
      }
      const float u0 = Ps[sc] * e0.x, tt = Ps[sc] * e0.y;
      const float2 uu = make_float2(u0, tt * e1.x);
      Ps[sc] = tt * e1.y;
      const float *qp = qh + pp * G * 2;
      if constexpr (G == 1) {
        acc[sc][0] = ffma2(uu, *reinterpret_cast<const float2 *>(qp), acc[sc][0]);
      } else {
#pragma unroll
        for (int g = 0; g < G; g += 2) {
          const float4 q4 = *reinterpret_cast<const float4 *>(qp + 2 * g);
          acc[sc][g] = ffma2(uu, make_float2(q4.x, q4.y), acc[sc][g]);
          acc[sc][g + 1] = ffma2(uu, make_float2(q4.z, q4.w), acc[sc][g + 1]);
        }
      }
    }
  }
  const float P1 = Ps[0], Pt = Ps[0] * Ps[1];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float A = fmaf(P1, acc[1][g].x + acc[1][g].y, acc[0][g].x + acc[0][g].y);
    const float Bh = __shfl_down_sync(0xffffffffu, A, 16);
    f[g] = fmaf(Pt, Bh, A);
  }
}

// f_b for two records (pages A and B of the same kv row and tier, b <= 4):
// lane (t, half) runs one chain of 64 fields for slot t of each page, and
// every query load serves both.  Results valid on lanes 0..15.
template <int BITS, int G, int QT_HALF>
__device__ __forceinline__ void ada_2page_f(const uint8_t *recA, const uint8_t *recB, const float *qt,
                                            const float2 *lpol, const float2 *laz, int lane, float (&fA)[G],
                                            float (&fB)[G]) {
  static_assert(BITS == 3 || BITS == 4, "pair path for b <= 4");
  const int t = lane & 15, half = lane >> 4;
  uint32_t W[2][2 * BITS];
#pragma unroll
  for (int pg = 0; pg < 2; ++pg) {
    const uint8_t *rec = pg ? recB : recA;
    if constexpr (BITS == 4) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint4 v = *reinterpret_cast<const uint4 *>(rec + ((half * 2 + k) * 16 + t) * 16);
        W[pg][4 * k + 0] = v.x;
        W[pg][4 * k + 1] = v.y;
        W[pg][4 * k + 2] = v.z;
        W[pg][4 * k + 3] = v.w;
      }
    } else {
      const uint4 A = *reinterpret_cast<const uint4 *>(rec + ((half + 0) * 16 + t) * 16);
      const uint4 Bv = *reinterpret_cast<const uint4 *>(rec + ((half + 1) * 16 + t) * 16);
      W[pg][0] = half ? A.z : A.x;
      W[pg][1] = half ? A.w : A.y;
      W[pg][2] = half ? Bv.x : A.z;
      W[pg][3] = half ? Bv.y : A.w;
      W[pg][4] = half ? Bv.z : Bv.x;
      W[pg][5] = half ? Bv.w : Bv.y;
    }
  }
  const float *qh = qt + half * QT_HALF;
  const float2 *l62 = half ? laz : lpol;
  float2 acc[2][G];
  float Ps[2] = {1.f, 1.f};
#pragma unroll
  for (int pg = 0; pg < 2; ++pg)
#pragma unroll
    for (int g = 0; g < G; ++g) acc[pg][g] = make_float2(0.f, 0.f);
#pragma unroll
  for (int pp = 0; pp < 32; ++pp) {
    float2 uu[2];
#pragma unroll
    for (int pg = 0; pg < 2; ++pg) {
      const uint32_t c0 = code_at<BITS>(W[pg], 2 * pp), c1 = code_at<BITS>(W[pg], 2 * pp + 1);
      float2 e0, e1;
      if (pp == 31) {
        e0 = l62[c0];
        const float2 t1 = lpol[half ? 0u : c1];
        e1 = make_float2(half ? 1.0f : t1.x, half ? 0.0f : t1.y);
      } else {
        e0 = lpol[c0];
        e1 = lpol[c1];
      }
      const float u0 = Ps[pg] * e0.x, tt = Ps[pg] * e0.y;
      uu[pg] = make_float2(u0, tt * e1.x);
      Ps[pg] = tt * e1.y;
    }
    const float *qp = qh + pp * G * 2;
    if constexpr (G == 1) {
      const float2 q2 = *reinterpret_cast<const float2 *>(qp);
      acc[0][0] = ffma2(uu[0], q2, acc[0][0]);
      acc[1][0] = ffma2(uu[1], q2, acc[1][0]);
    } else {
#pragma unroll
      for (int g = 0; g < G; g += 2) {
        const float4 q4 = *reinterpret_cast<const float4 *>(qp + 2 * g);
        const float2 qa = make_float2(q4.x, q4.y), qb = make_float2(q4.z, q4.w);
        acc[0][g] = ffma2(uu[0], qa, acc[0][g]);
        acc[0][g + 1] = ffma2(uu[0], qb, acc[0][g + 1]);
        acc[1][g] = ffma2(uu[1], qa, acc[1][g]);
        acc[1][g + 1] = ffma2(uu[1], qb, acc[1][g + 1]);
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float Aa = acc[0][g].x + acc[0][g].y, Ab = acc[1][g].x + acc[1][g].y;
    const float Ba = __shfl_down_sync(0xffffffffu, Aa, 16), Bb = __shfl_down_sync(0xffffffffu, Ab, 16);
    fA[g] = fmaf(Ps[0], Ba, Aa);
    fB[g] = fmaf(Ps[1], Bb, Ab);
  }
}

// b = 4 version of ada_2page_f with a rolled loop: each iteration decodes the
// 16 pairs of one 16-byte code chunk (32 fields) of both pages, so the loop
// body (and the instruction footprint) is half of the unrolled one.  The
// (cos, sin) table of b = 4 is 16 float2 = one 128-byte row starting at a
// 256-byte aligned shared address.  Each code word is spread once into
// bytes holding 8 x code (even fields in E, odd fields in O); a field's entry
// address is then one byte permute: the entry offset as the low byte under
// the table's upper address bytes.  NIT = 4 or 8 shortens the body further
// (16 or 8 fields, two words or one per page and iteration): measured faster
// for G = 8 (NIT = 4) and in the mixed-tier kernel (NIT = 8), whose warps run
// several tiers' paths at once; slower for G <= 4 on a b = 4 cache.
template <int G, int QT_HALF, int NIT = 2>
__device__ __forceinline__ void ada_2page_f4(const uint8_t *recA, const uint8_t *recB, const float *qt,
                                             uint32_t lpol_s, uint32_t laz_s, int lane, float (&fA)[G],
                                             float (&fB)[G]) {
  static_assert(NIT == 2 || NIT == 4 || NIT == 8, "32, 16 or 8 fields per iteration");
  constexpr int PPI = 32 / NIT, NWD = 8 / NIT;  // pairs and code words per page and iteration
  const int t = lane & 15, half = lane >> 4;
  const float *qh = qt + half * QT_HALF;
  float2 acc[2][G];
  float Ps[2] = {1.f, 1.f};
#pragma unroll
  for (int pg = 0; pg < 2; ++pg)
#pragma unroll
    for (int g = 0; g < G; ++g) acc[pg][g] = make_float2(0.f, 0.f);
#pragma unroll 1
  for (int it = 0; it < NIT; ++it) {
    uint32_t WA[NWD], WB[NWD];
    if constexpr (NIT == 2) {
      const int chunk = half * 2 + it;
      const uint4 wa = *reinterpret_cast<const uint4 *>(recA + (chunk * 16 + t) * 16);
      const uint4 wb = *reinterpret_cast<const uint4 *>(recB + (chunk * 16 + t) * 16);
      WA[0] = wa.x; WA[1] = wa.y; WA[2] = wa.z; WA[3] = wa.w;
      WB[0] = wb.x; WB[1] = wb.y; WB[2] = wb.z; WB[3] = wb.w;
    } else if constexpr (NIT == 4) {  // words 2 (it & 1), +1 of chunk 2 half + it / 2
      const int off = ((half * 2 + (it >> 1)) * 16 + t) * 16 + (it & 1) * 8;
      const uint2 wa = *reinterpret_cast<const uint2 *>(recA + off);
      const uint2 wb = *reinterpret_cast<const uint2 *>(recB + off);
      WA[0] = wa.x; WA[1] = wa.y;
      WB[0] = wb.x; WB[1] = wb.y;
    } else {  // word it & 3 of chunk 2 half + it / 4
      const int off = ((half * 2 + (it >> 2)) * 16 + t) * 16 + (it & 3) * 4;
      WA[0] = *reinterpret_cast<const uint32_t *>(recA + off);
      WB[0] = *reinterpret_cast<const uint32_t *>(recB + off);
    }
    // the iteration's last pair is (azimuth, padding) in the second half
    const bool tail = it == NIT - 1 && half;
    const float *qi = qh + it * PPI * G * 2;
#pragma unroll
    for (int pq = 0; pq < PPI; ++pq) {
      float2 uu[2];
#pragma unroll
      for (int pg = 0; pg < 2; ++pg) {
        const uint32_t w = pg ? WB[pq >> 2] : WA[pq >> 2];
        const uint32_t ev = (w << 3) & 0x78787878u, od = (w >> 1) & 0x78787878u;  // CSE'd per word
        const uint32_t sel = 0x7650u | (uint32_t)(pq & 3);
        float2 e0, e1;
        if (pq == PPI - 1) {
          e0 = lds_f2(__byte_perm(ev, tail ? laz_s : lpol_s, sel));
          const float2 t1 = lds_f2(__byte_perm(od, lpol_s, sel));
          e1 = make_float2(tail ? 1.0f : t1.x, tail ? 0.0f : t1.y);
        } else {
          e0 = lds_f2(__byte_perm(ev, lpol_s, sel));
          e1 = lds_f2(__byte_perm(od, lpol_s, sel));
        }
        const float u0 = Ps[pg] * e0.x, tt = Ps[pg] * e0.y;
        uu[pg] = make_float2(u0, tt * e1.x);
        Ps[pg] = tt * e1.y;
      }
      const float *qp = qi + pq * G * 2;
      if constexpr (G == 1) {
        const float2 q2 = *reinterpret_cast<const float2 *>(qp);
        acc[0][0] = ffma2(uu[0], q2, acc[0][0]);
        acc[1][0] = ffma2(uu[1], q2, acc[1][0]);
      } else {
#pragma unroll
        for (int g = 0; g < G; g += 2) {
          const float4 q4 = *reinterpret_cast<const float4 *>(qp + 2 * g);
          const float2 qa = make_float2(q4.x, q4.y), qb = make_float2(q4.z, q4.w);
          acc[0][g] = ffma2(uu[0], qa, acc[0][g]);
          acc[0][g + 1] = ffma2(uu[0], qb, acc[0][g + 1]);
          acc[1][g] = ffma2(uu[1], qa, acc[1][g]);
          acc[1][g + 1] = ffma2(uu[1], qb, acc[1][g + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float Aa = acc[0][g].x + acc[0][g].y, Ab = acc[1][g].x + acc[1][g].y;
    const float Ba = __shfl_down_sync(0xffffffffu, Aa, 16), Bb = __shfl_down_sync(0xffffffffu, Ab, 16);
    fA[g] = fmaf(Ps[0], Ba, Aa);
    fB[g] = fmaf(Ps[1], Bb, Ab);
  }
}

// Pair path for any width b (used for b = 3, 6, 8 in the mixed-tier kernel;
// b = 4 has ada_2page_f4): a rolled loop over the 64 fields of the lane's
// half, eight iterations of 8 fields of both pages -- 8 b bits of the slot's
// stream, two words per page loaded and shifted into place per iteration --
// so the loop body stays short (the mixed-tier kernel was bound by
// instruction fetch: each shortening of this body measured faster).
template <int BITS, int G, int QT_HALF>
__device__ __forceinline__ void ada_2page_gen(const uint8_t *recA, const uint8_t *recB, const float *qt,
                                              const float2 *lpol, const float2 *laz, int lane, float (&fA)[G],
                                              float (&fB)[G]) {
  constexpr int NIT = 8;
  constexpr int FPI = 64 / NIT, PPI = FPI / 2, WPI = 2;  // fields, pairs, words per iteration
  const uint32_t lpol_s = smem_u32(lpol), laz_s = smem_u32(laz);
  const int t = lane & 15, half = lane >> 4;
  const float *qh = qt + half * QT_HALF;
  const uint32_t *ra32 = reinterpret_cast<const uint32_t *>(recA);
  const uint32_t *rb32 = reinterpret_cast<const uint32_t *>(recB);
  float2 acc[2][G];
  float Ps[2] = {1.f, 1.f};
#pragma unroll
  for (int pg = 0; pg < 2; ++pg)
#pragma unroll
    for (int g = 0; g < G; ++g) acc[pg][g] = make_float2(0.f, 0.f);
#pragma unroll 1
  for (int it = 0; it < NIT; ++it) {
    // word w of the stream: chunk w / 4, word w % 4 of the slot's 16 bytes
    auto word = [&](const uint32_t *r32, int w) { return r32[(16 * (w >> 2) + t) * 4 + (w & 3)]; };
    uint32_t WA[WPI], WB[WPI];
    {  // bits [8 b it, 8 b it + 8 b) of the half's 64 b, from two words shifted into place:
       // sh + 8 b <= 64 (sh in {0, 8, 16, 24} for b = 3, {0, 16} for b = 6, 0 for b = 8);
       // the second word is clamped to the slot's last (its bits are then unused)
      static_assert(BITS == 3 || BITS == 6 || BITS == 8, "widths of the pair path");
      const int bit0 = it * FPI * BITS, w0 = 2 * half * BITS + (bit0 >> 5), sh = bit0 & 31;
      const int w1 = w0 + 1 < 4 * BITS ? w0 + 1 : w0;
      const uint64_t a = ((uint64_t)word(ra32, w1) << 32 | word(ra32, w0)) >> sh;
      const uint64_t b = ((uint64_t)word(rb32, w1) << 32 | word(rb32, w0)) >> sh;
      WA[0] = (uint32_t)a;
      WA[1] = (uint32_t)(a >> 32);
      WB[0] = (uint32_t)b;
      WB[1] = (uint32_t)(b >> 32);
    }
    const bool tail = it == NIT - 1 && half;  // the iteration's last pair is (azimuth, padding)
    const float *qi = qh + it * PPI * G * 2;
#pragma unroll
    for (int pq = 0; pq < PPI; ++pq) {
      float2 uu[2];
#pragma unroll
      for (int pg = 0; pg < 2; ++pg) {
        const uint32_t o0 = off8_at<BITS, WPI>(pg ? WB : WA, 2 * pq * BITS);
        const uint32_t o1 = off8_at<BITS, WPI>(pg ? WB : WA, (2 * pq + 1) * BITS);
        float2 e0, e1;
        if (pq == PPI - 1) {
          e0 = lds_f2((tail ? laz_s : lpol_s) + o0);
          const float2 t1 = lds_f2(lpol_s + o1);
          e1 = make_float2(tail ? 1.0f : t1.x, tail ? 0.0f : t1.y);
        } else {
          e0 = lds_f2(lpol_s + o0);
          e1 = lds_f2(lpol_s + o1);
        }
        const float u0 = Ps[pg] * e0.x, tt = Ps[pg] * e0.y;
        uu[pg] = make_float2(u0, tt * e1.x);
        Ps[pg] = tt * e1.y;
      }
      const float *qp = qi + pq * G * 2;
      if constexpr (G == 1) {
        const float2 q2 = *reinterpret_cast<const float2 *>(qp);
        acc[0][0] = ffma2(uu[0], q2, acc[0][0]);
        acc[1][0] = ffma2(uu[1], q2, acc[1][0]);
      } else {
#pragma unroll
        for (int g = 0; g < G; g += 2) {
          const float4 q4 = *reinterpret_cast<const float4 *>(qp + 2 * g);
          const float2 qa = make_float2(q4.x, q4.y), qb = make_float2(q4.z, q4.w);
          acc[0][g] = ffma2(uu[0], qa, acc[0][g]);
          acc[0][g + 1] = ffma2(uu[0], qb, acc[0][g + 1]);
          acc[1][g] = ffma2(uu[1], qa, acc[1][g]);
          acc[1][g + 1] = ffma2(uu[1], qb, acc[1][g + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float Aa = acc[0][g].x + acc[0][g].y, Ab = acc[1][g].x + acc[1][g].y;
    const float Ba = __shfl_down_sync(0xffffffffu, Aa, 16), Bb = __shfl_down_sync(0xffffffffu, Ab, 16);
    fA[g] = fmaf(Ps[0], Ba, Aa);
    fB[g] = fmaf(Ps[1], Bb, Ab);
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
// Workspace: one partial record (m, l, pad, pad, acc[128]) per query head for
// every (split c, kv-head row bh) segment and consumer warp w, at
// ws + (((c + bh) * NCW + w) * G + g) * 132 floats (NCW consumer warps of
// the path); m is in log2 units.
constexpr int kPartial = 132;

// Fused single-token append, by the producer warp: the new key of kv row
// (b, h) -- token ctx_lens[b] - 1, the last one of the row's last page pid,
// whose record (width `bits`) starts at byte rec_off of the arena -- is
// encoded into its slot exactly as spkv_encode_keys would write it, and the
// new value row goes to the same slot of the value page.  Called before the
// page's copy is issued; the caller fences the stores for the async proxy.
__device__ __noinline__ void append_token(const SplitParams &p, int b, int h, int pid, int bits, uint64_t rec_off,
                                          const double *pol_c2, const double *az_c2, int lane) {
  const int slot = (p.ctx_lens[b] - 1) % kPage;
  const int64_t row = (int64_t)b * p.Hkv + h;
  // the key: the warp form of spkv_encode_keys' arithmetic (the same bytes)
  encode_key_warp_seq_bits(bits, p.new_k + row * kD, const_cast<uint8_t *>(p.arena) + rec_off, slot, p.rad_lo[h],
                           p.rad_step[h], pol_c2, az_c2, lane, p.err);
  const uint2 v = *reinterpret_cast<const uint2 *>(p.new_v + row * kD + 4 * lane);
  *reinterpret_cast<uint2 *>(const_cast<uint16_t *>(p.v_pages) + (((int64_t)pid * p.Hkv + h) * kPage + slot) * kD +
                             4 * lane) = v;
  __syncwarp();
}

template <bool ADA, int G, bool NW>
__global__ void __launch_bounds__(Layout<ADA, G, NW>::THREADS, 2)
    split_kernel(const SplitParams p, const __grid_constant__ CUtensorMap vmap) {
  using Ly = Layout<ADA, G, NW>;
  constexpr int NCW = Ly::NCW, NST = Ly::NST;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t *vslot_all = smem + Ly::off_v;
  uint8_t *xst_all = smem + Ly::off_x;
  float2 *lpol = reinterpret_cast<float2 *>(smem + Ly::off_lut);
  float2 *laz = lpol + Ly::LAZ_OFF;
  float *qt = reinterpret_cast<float *>(smem + Ly::off_qt);
  // fp64 edge tables of the exact code decisions (query coding, fused append),
  // built once per CTA
  double *pol_c2 = reinterpret_cast<double *>(smem + Ly::off_pe);
  double *az_c2 = pol_c2 + kLutEntries;
  float *pbuf_all = reinterpret_cast<float *>(smem + Ly::off_pbuf);
  float *sc = reinterpret_cast<float *>(smem + Ly::off_sc);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + Ly::off_bar);
  uint64_t *empty = full + NST;
  uint64_t *vbar_all = empty + NST;  // 1 per consumer warp
  StageMeta *meta = reinterpret_cast<StageMeta *>(smem + Ly::off_meta);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Ly::off_misc);
  int32_t *scratch = reinterpret_cast<int32_t *>(smem + Ly::off_misc + 16);
  int32_t *P = reinterpret_cast<int32_t *>(smem + Ly::off_P);

  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int C = gridDim.x, c = blockIdx.x;

  // the merge grid may be launched now: its blocks only take SMs that this
  // grid's CTAs leave, and each waits for the rows it merges
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  build_prefix(p.ctx_lens, p.B, p.Hkv, p.max_ctx, p.max_pages, p.err, P, scratch, tid, Ly::THREADS);
  const Partition part(P, p.B, p.Hkv, C);
  const int64_t u0 = part.begin(c), u1 = part.begin(c + 1);
  if (u0 >= u1) return;  // uniform across the block

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int v = 0; v < NCW; ++v) mbar_init(&vbar_all[v], 1);
    if (ADA) mbar_init(&vbar_all[NCW], 1);  // the consumers' tables are built (a spare slot)
    *abort_flag = 0;
    mbar_fence_init();
  }

  __syncthreads();

  const int n_units = (int)(u1 - u0);

  if (wid == NCW) {
    // =========================== producer warp ===========================
    // Unit k (CTA-relative) goes to stage k % NST.  Metadata of a batch of 32
    // units is fetched by the 32 lanes in two dependent rounds (block table,
    // then header / mask), half a batch ahead.
    struct A_ {
      int pid, ntok, h, ok, last, b;
    };
    struct B_ {
      uint32_t off16;
      int bits;
      uint32_t keep;
    };
    // units [u0 + kb + lane] below CTA-relative unit `lim`
    auto phaseA = [&](int kb, int lim) -> A_ {
      A_ a{0, 0, 0, 0, 0, 0};
      const int k = kb + lane;
      if (k < lim) {
        const int64_t u = u0 + k;
        const int b = find_seq(P, p.B, u);
        const int np = (P[b + 1] - P[b]) / p.Hkv;
        const int rem = (int)(u - P[b]);
        const int h = rem / np, j = rem - h * np;
        a.h = h;
        a.pid = p.block_table[(int64_t)b * p.max_pages + j];
        const int ctx = p.ctx_lens[b];
        a.ntok = min(kPage, ctx - j * kPage);
        a.last = j == np - 1;
        a.b = b;
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
    // a unit's copy plan: checks (flagging bad pages), record and value offsets
    struct U_ {
      int valid;
      uint64_t rec_off, v_off;
      uint32_t rec_sz, live;
    };
    auto plan = [&](const A_ &ac, const B_ &bc) -> U_ {
      U_ x{0, 0, 0, 0, 0};
      if (ac.ok) {
        const int ti = tier_of_bits(bc.bits);
        if (ac.pid < 0 || ac.pid >= p.num_pages) {
          set_err(p.err, SPKV_DEVERR_PAGE_ID);
        } else if (ADA && (ti < 0 || !((p.tiers >> ti) & 1u))) {
          set_err(p.err, SPKV_DEVERR_BITS);
        } else {
          x.v_off = ((uint64_t)ac.pid * p.Hkv + ac.h) * (kPage * kD);
          if constexpr (ADA) {
            x.rec_sz = rec_bytes(bc.bits);
            x.rec_off = (uint64_t)bc.off16 * 16u + (uint64_t)ac.h * x.rec_sz;
            if (x.rec_off + x.rec_sz > p.arena_bytes) set_err(p.err, SPKV_DEVERR_RECORD);
            else x.valid = 1;
          } else {
            x.valid = 1;
          }
        }
      }
      x.live = bc.keep & ((1u << ac.ntok) - 1u);
      return x;
    };
    bool tables = false;
    // One issue step (warp-wide): the lanes with `mine` set fill their units'
    // stages s = k % NST (at most kIssue distinct stages per step).
    auto issue = [&](const A_ &ac, const B_ &bc, const U_ &x, bool mine, int k) {
      const int s = k % NST, r = k / NST;
      if constexpr (ADA) {
        // fused append: a row's last page gets the step's token before its copy
        uint32_t todo = p.new_k ? __ballot_sync(0xffffffffu, mine && x.valid && ac.last) : 0u;
        if (todo) {
          if (!tables) {  // the fused append codes with the consumers' edge tables
            mbar_wait_sleepy(&vbar_all[NCW], 0u, abort_flag, p.err);
            tables = true;
          }
          while (todo) {
            const int src = __ffs(todo) - 1;
            todo &= todo - 1;
            append_token(p, __shfl_sync(0xffffffffu, ac.b, src), __shfl_sync(0xffffffffu, ac.h, src),
                         __shfl_sync(0xffffffffu, ac.pid, src), __shfl_sync(0xffffffffu, bc.bits, src),
                         __shfl_sync(0xffffffffu, x.rec_off, src), pol_c2, az_c2, lane);
          }
          // the copies below (and the consumers' value TMA) read what was written
          __threadfence();
          asm volatile("fence.proxy.async.global;" ::: "memory");
          __syncwarp();
        }
      }
      if (mine) {
        if (r > 0) mbar_wait_sleepy(&empty[s], (uint32_t)(r - 1) & 1u, abort_flag, p.err);
        StageMeta m;
        m.valid = x.valid && !*abort_flag;
        m.bits = bc.bits;
        m.ntok = ac.ntok;
        m.live = x.live;
        m.vrow = (int)(x.v_off / kD);  // (pid * H_kv + h) * 16
        meta[s] = m;
        uint8_t *xst = xst_all + s * Ly::XSTAGE;
        if (m.valid) {
          if constexpr (ADA) {
            mbar_arrive_expect_tx(&full[s], x.rec_sz);
            bulk_g2s(xst, p.arena + x.rec_off, x.rec_sz, &full[s]);
          } else {
            mbar_arrive_expect_tx(&full[s], 4096u);
            bulk_g2s(xst, p.k_pages + x.v_off, 4096u, &full[s]);
          }
        } else {
          mbar_arrive(&full[s]);
        }
      }
      __syncwarp();
    };
    int k_last = -1;
    if (ADA && !NW && __popc(p.tiers) > 1) {
      // Several tiers (wide caches; a narrow cache's b = 3 and b = 4 both pair): a kv row's pages may be decoded in any order (softmax
      // and P.V run over the set), so each segment is walked once per tier
      // present and that tier's pages take the next units.  Long runs of one
      // tier keep neighbouring units paired and every warp on one code path.
      // (Pages whose header names no tier of the mask go with the first pass,
      // as units the consumers skip.)
      const int t_first = __ffs(p.tiers) - 1;
      int next_k = 0;
      int sa = 0;
      while (sa < n_units) {
        const int64_t ua = u0 + sa;
        const int b = find_seq(P, p.B, ua);
        const int np = (P[b + 1] - P[b]) / p.Hkv;
        const int h = (int)((ua - P[b]) / np);
        const int64_t seg_hi = (int64_t)P[b] + (int64_t)(h + 1) * np;
        const int se = (int)((seg_hi < u1 ? seg_hi : u1) - u0);
        for (int t = t_first; t < kTiers; ++t) {
          if (!((p.tiers >> t) & 1u)) continue;
          for (int sb = sa; sb < se; sb += 32) {
            const A_ ac = phaseA(sb, se);
            const B_ bc = phaseB(ac);
            const U_ x = plan(ac, bc);
            const int ti = tier_of_bits(bc.bits);
            const bool in_mask = ti >= 0 && ((p.tiers >> ti) & 1u);
            const bool sel = ac.ok && (in_mask ? ti == t : t == t_first);
            const uint32_t sm = __ballot_sync(0xffffffffu, sel);
            const int rank = __popc(sm & ((1u << lane) - 1u)), nsel = __popc(sm);
            for (int i0 = 0; i0 < nsel; i0 += kIssue)
              issue(ac, bc, x, sel && rank >= i0 && rank < i0 + kIssue, next_k + rank);
            next_k += nsel;
          }
        }
        sa = se;
      }
      k_last = next_k - 1;
    } else {
      A_ an = phaseA(0, n_units);
      B_ bn = phaseB(an);
      for (int kb = 0; kb < n_units; kb += 32) {
        const A_ ac = an;
        const B_ bc = bn;
        int valid = 0;
        uint64_t rec_off = 0, v_off = 0;
        uint32_t rec_sz = 0;
        if (ac.ok) {
          const int ti = tier_of_bits(bc.bits);
          if (ac.pid < 0 || ac.pid >= p.num_pages) {
            set_err(p.err, SPKV_DEVERR_PAGE_ID);
          } else if (ADA && (ti < 0 || !((p.tiers >> ti) & 1u))) {
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
        an = phaseA(kb + 32, n_units);
        const int cnt = min(32, n_units - kb);
        // lanes [i0, i0 + kIssue) wait for their own stages and issue together
        for (int i0 = 0; i0 < cnt; i0 += kIssue) {
          if (i0 == 16) bn = phaseB(an);
          const int k = kb + lane, s = k % NST, r = k / NST;
          const bool mine = lane >= i0 && lane < i0 + kIssue && lane < cnt;
          if constexpr (ADA) {
            // fused append: a row's last page gets the step's token before its copy
            uint32_t todo = p.new_k ? __ballot_sync(0xffffffffu, mine && valid && ac.last) : 0u;
            if (todo) {
              if (!tables) {  // the fused append codes with the consumers' edge tables
                mbar_wait_sleepy(&vbar_all[NCW], 0u, abort_flag, p.err);
                tables = true;
              }
              while (todo) {
                const int src = __ffs(todo) - 1;
                todo &= todo - 1;
                append_token(p, __shfl_sync(0xffffffffu, ac.b, src), __shfl_sync(0xffffffffu, ac.h, src),
                             __shfl_sync(0xffffffffu, ac.pid, src), __shfl_sync(0xffffffffu, bc.bits, src),
                             __shfl_sync(0xffffffffu, rec_off, src), pol_c2, az_c2, lane);
              }
              // the copies below (and the consumers' value TMA) read what was written
              __threadfence();
              asm volatile("fence.proxy.async.global;" ::: "memory");
              __syncwarp();
            }
          }
          if (mine) {
            if (r > 0) mbar_wait_sleepy(&empty[s], (uint32_t)(r - 1) & 1u, abort_flag, p.err);
            StageMeta m;
            m.valid = valid && !*abort_flag;
            m.bits = bc.bits;
            m.ntok = ac.ntok;
            m.live = live;
            m.vrow = (int)(v_off / kD);  // (pid * H_kv + h) * 16
            meta[s] = m;
            uint8_t *xst = xst_all + s * Ly::XSTAGE;
            if (m.valid) {
              if constexpr (ADA) {
                mbar_arrive_expect_tx(&full[s], rec_sz);
                bulk_g2s(xst, p.arena + rec_off, rec_sz, &full[s]);
              } else {
                mbar_arrive_expect_tx(&full[s], 4096u);
                bulk_g2s(xst, p.k_pages + v_off, 4096u, &full[s]);
              }
            } else {
              mbar_arrive(&full[s]);
            }
          }
          __syncwarp();
        }
        k_last = kb + cnt - 1;
        if (cnt <= 16) bn = phaseB(an);
      }
    }
    // On an abort, copies may still be in flight into our stages: wait for
    // them (bounded) before the CTA's shared memory can be released.
    if (*abort_flag && lane == 0) {
      volatile int dummy = 0;
      for (int s = 0; s < NST; ++s) {
        const int kk = k_last - ((k_last - s) % NST + NST) % NST;  // last unit in stage s
        if (kk >= 0) mbar_wait_bounded(&full[s], (uint32_t)(kk / NST) & 1u, &dummy, nullptr);
      }
    }
    return;
  }

  // ============================= consumer warps ============================
  // Units are grouped in pairs (2i, 2i + 1); pair i belongs to warp i % NCW.
  // A pair whose two units lie in one segment and share a tier b <= 4 is
  // decoded in one pass (every query load serves both pages); any other
  // unit is decoded on its own.
  float *pbuf = pbuf_all + wid * (G * 2 * kPage);
  const int grp = lane >> 2, tig = lane & 3;
  uint8_t *const vslot[2] = {vslot_all + (2 * wid) * Ly::VSLOT, vslot_all + (2 * wid + 1) * Ly::VSLOT};
  uint64_t *const vbar = vbar_all + wid;  // the value pages of this warp's pair
  uint32_t vphase = 0u;
  int vpending = -1;  // phase of a value load a failed wait left in flight
  if constexpr (ADA) {  // the consumers' tables, while the producer starts the ring
    build_luts(lpol, laz, tid, NCW * 32);
    build_edge_tables(pol_c2, az_c2, tid, NCW * 32);
    named_bar_sync(1, NCW * 32);
    if (tid == 0) mbar_arrive(&vbar_all[NCW]);
  }
  int64_t u = u0;
  while (u < u1) {
    const int b = find_seq(P, p.B, u);
    const int np = (P[b + 1] - P[b]) / p.Hkv;
    const int h = (int)((u - P[b]) / np);
    const int64_t seg_hi = (int64_t)P[b] + (int64_t)(h + 1) * np;
    const int64_t seg_end = seg_hi < u1 ? seg_hi : u1;
    const int bh = b * p.Hkv + h;

    // ---- per-segment query preparation (every consumer warp is past the
    // previous segment's last page: the query table may be rewritten)
    named_bar_sync(1, NCW * 32);
    for (int g = wid; g < G; g += NCW) {
      const uint16_t *qrow = p.q + ((int64_t)b * p.Hq + (int64_t)h * G + g) * kD;
      if constexpr (ADA) {
        const float qn = ada_qprep_row<G, Ly::QT_HALF>(qrow, g, lpol, laz, pol_c2, az_c2, qt, lane, p.tiers,
                                                       (p.flags & SPKV_DECODE_EXACT_Q) != 0u);
        if (lane == 0) sc[g] = qn * kLog2e * 0.08838834764831845f;
      } else {
        dense_qprep_row<G, Ly::QT_HALF>(qrow, g, qt, lane);
      }
    }
    if constexpr (ADA) {
      if (tid == 0) {
        sc[G] = p.rad_lo[h];
        sc[G + 1] = p.rad_step[h];
      }
    }
    named_bar_sync(1, NCW * 32);

    float m[G], lsum[G];
    // P.V accumulators in m16n8k16 fragment layout (D^T = V^T P^T):
    // d[mb][0..1] = dim 16 mb + grp, columns 2 tig, 2 tig + 1; d[mb][2..3] = dim + 8.
    // Column c is head c (G = 8: P hi and lo in two MMAs), or for G <= 4 the
    // hi part of head c (c < G) and the lo part of head c - G (G <= c < 2G).
    constexpr bool kPackPV = G <= 4;
    float d[8][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = kNegInf;
      lsum[g] = 0.f;
    }
#pragma unroll
    for (int mb = 0; mb < 8; ++mb) d[mb][0] = d[mb][1] = d[mb][2] = d[mb][3] = 0.f;
    float scg[G];
#pragma unroll
    for (int g = 0; g < G; ++g) scg[g] = sc[g];
    const float Lh = ADA ? sc[G] : 0.f, Dh = ADA ? sc[G + 1] : 0.f;

    // logits of a page (ADA from codes, narrow ring; dense from bf16 keys), lanes 0..15
    auto page_logits = [&](const StageMeta &mt, const uint8_t *xst, float (&l2)[G]) {
      if constexpr (ADA) {
        float f[G];
        const int ti = tier_of_bits(mt.bits);
        const float *q0 = qt + ti * Ly::QT_TIER;
        const float2 *lp = lpol + lut_off(ti), *la = laz + lut_off(ti);
        // (narrow ring only: the producer admits no page of b > 4 into it;
        // the two forms below compile to faster code for their G)
        if constexpr (G == 8) {
          if (mt.bits == 4) ada_page_f<4, G, Ly::QT_HALF>(xst, q0, lp, la, lane, f);
          else ada_page_f<3, G, Ly::QT_HALF>(xst, q0, lp, la, lane, f);
        } else {
          switch (mt.bits) {
            case 3: ada_page_f<3, G, Ly::QT_HALF>(xst, q0, lp, la, lane, f); break;
            case 4: ada_page_f<4, G, Ly::QT_HALF>(xst, q0, lp, la, lane, f); break;
            default: break;
          }
        }
        const float rad = fast_exp2(fmaf((float)xst[256 * mt.bits + (lane & 15)], Dh, Lh));
#pragma unroll
        for (int g = 0; g < G; ++g) l2[g] = scg[g] * rad * f[g];
      } else {
        dense_page_logits<G, Ly::QT_HALF>(xst, qt, lane, l2);
      }
    };

    // online softmax over the pages of a pair (slots 0..15 and 16..31 of
    // pbuf; use[q] = 0 drops page q) followed by P.V on tensor cores.  The
    // running max m only moves when a page's max exceeds it by more than
    // kRescaleSlack, so p <= 2^8 and the accumulators are rescaled on few pages.
    auto softmax_pv = [&](const bool (&use)[2], const StageMeta (&mt)[2], const float (&l2)[2][G],
                          uint8_t *const (&vs)[2]) {
      float x[2][G];
      bool alive[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        alive[q] = use[q] && lane < 16 && ((mt[q].live >> (lane & 15)) & 1u);
#pragma unroll
        for (int g = 0; g < G; ++g) x[q][g] = alive[q] ? l2[q][g] : kNegInf;
      }
      bool moved = false;
      float alpha[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float xm = fmaxf(x[0][g], x[1][g]);
        alpha[g] = 1.f;
        // the warp max exceeds m + slack iff some lane's does (one vote on
        // the common path; the max itself only when m moves)
        if (__any_sync(0xffffffffu, xm > m[g] + kRescaleSlack)) {
          const float mx = warp_max(xm);
          alpha[g] = m[g] == kNegInf ? 0.f : fast_exp2(m[g] - mx);
          m[g] = mx;
          moved = true;
        }
        const float pa = (alive[0] && m[g] != kNegInf) ? fast_exp2(x[0][g] - m[g]) : 0.f;
        const float pb = (alive[1] && m[g] != kNegInf) ? fast_exp2(x[1][g] - m[g]) : 0.f;
        lsum[g] = fmaf(lsum[g], alpha[g], pa + pb);
        if (lane < 16) {
          pbuf[g * 2 * kPage + lane] = pa;
          pbuf[g * 2 * kPage + kPage + lane] = pb;
        }
      }
      if (moved) {  // rescale the fragments of columns 2 tig, 2 tig + 1
        float a0 = 1.f, a1 = 1.f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (2 * tig == g || (kPackPV && 2 * tig == g + G)) a0 = alpha[g];
          if (2 * tig + 1 == g || (kPackPV && 2 * tig + 1 == g + G)) a1 = alpha[g];
        }
#pragma unroll
        for (int mb = 0; mb < 8; ++mb) {
          d[mb][0] *= a0;
          d[mb][1] *= a1;
          d[mb][2] *= a0;
          d[mb][3] *= a1;
        }
      }
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (!use[q]) continue;  // warp-uniform
        // rows past the context end (last page) may hold anything: zero them
        // so that p = 0 times the row stays 0
        if (mt[q].ntok < kPage) {
          for (int i = lane; i < (kPage - mt[q].ntok) * 16; i += 32) {
            const int row = mt[q].ntok + (i >> 4), box = (i >> 3) & 1, ch = i & 7;
            *reinterpret_cast<uint4 *>(vs[q] + box * 2048 + row * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        // B = P^T (16 slots x heads) as bf16 hi + lo: for G <= 4 the hi parts
        // are columns 0..G-1 and the lo parts columns G..2G-1 of one tile
        uint32_t bh0 = 0u, bh1 = 0u, bl0 = 0u, bl1 = 0u;
        const int hg = (kPackPV && grp >= G) ? grp - G : grp;
        if (hg < G) {
          const float *pr = pbuf + hg * 2 * kPage + q * kPage;
          const float2 pa = *reinterpret_cast<const float2 *>(pr + 2 * tig);
          const float2 pb = *reinterpret_cast<const float2 *>(pr + 2 * tig + 8);
          split_bf16x2(pa.x, pa.y, bh0, bl0);
          split_bf16x2(pb.x, pb.y, bh1, bl1);
          if (kPackPV && grp >= G) {
            bh0 = bl0;
            bh1 = bl1;
          }
        }
        const int vt = (lane & 7) + 8 * (lane >> 4);  // value row (slot) this lane addresses
        const uint32_t vrow = smem_u32(vs[q]) + (uint32_t)(vt * 128);
        const uint32_t jsel = (lane >> 3) & 1u, t7 = (uint32_t)(vt & 7);
#pragma unroll
        for (int mb = 0; mb < 8; ++mb) {
          uint32_t a[4];
          const uint32_t j = 2u * (uint32_t)(mb & 3) + jsel;  // 16-byte chunk within the box row
          ldsm_x4_trans(a, vrow + (uint32_t)(mb >> 2) * 2048u + ((j ^ t7) << 4));
          mma_bf16_16816(d[mb], a, bh0, bh1);
          if (!kPackPV) mma_bf16_16816(d[mb], a, bl0, bl1);
        }
      }
    };

    // ---- this segment's units: CTA-relative [ks, ke)
    const int ks = (int)(u - u0), ke = (int)(seg_end - u0);
    int i = ks >> 1;
    i += ((wid - i) % NCW + NCW) % NCW;
    // ready[q]: unit q of this warp's next pair was seen complete one pair
    // early (a non-blocking test whose latency hides behind the pair's work)
    bool ready[2] = {false, false};
    for (; 2 * i < ke; i += NCW) {
      const int ka = 2 * i < ks ? ks : 2 * i;
      const int kz = 2 * i + 2 > ke ? ke : 2 * i + 2;  // units [ka, kz) of pair i in this segment
      const int n = kz - ka;
      StageMeta mt[2];
      const uint8_t *xst[2];
      bool use[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        use[q] = false;
        xst[q] = xst_all;
        mt[q] = StageMeta{};
        if (q < n) {
          const int k = ka + q, s = k % NST;
          const bool ok = ready[q] || mbar_wait_bounded(&full[s], (uint32_t)(k / NST) & 1u, abort_flag, p.err);
          mt[q] = meta[s];
          use[q] = ok && mt[q].valid && mt[q].live;
          xst[q] = xst_all + s * Ly::XSTAGE;
        }
      }
      // the pair's value pages, into this warp's slots (overlaps the logits)
      const bool vload = use[0] || use[1];
      if (lane == 0 && vload) {
        mbar_arrive_expect_tx(vbar, 4096u * ((use[0] ? 1u : 0u) + (use[1] ? 1u : 0u)));
#pragma unroll
        for (int q = 0; q < 2; ++q)
          if (use[q]) tma_load_3d(vslot[q], &vmap, 0, mt[q].vrow, 0, vbar);
      }
      float l2[2][G];
      if constexpr (ADA && !NW) {
        // Wide ring (pages of every tier): one f_b call site, for a smaller
        // instruction footprint (warps of one SM run different tiers' paths
        // at once): a pair of one tier in one pass; otherwise each used page
        // alone, given as both pages of its pass.
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int g = 0; g < G; ++g) l2[q][g] = 0.f;
        const bool paired = use[0] && use[1] && mt[0].bits == mt[1].bits;
        const int npass = paired ? 1 : 2;
#pragma unroll 1
        for (int pass = 0; pass < npass; ++pass) {
          const int qa = paired ? 0 : pass, qb = paired ? 1 : pass;
          if (!(qa ? use[1] : use[0])) continue;  // warp-uniform
          float fa[G], fb[G];
          const int bits = qa ? mt[1].bits : mt[0].bits;
          const int ti = tier_of_bits(bits);
          const float *q0 = qt + ti * Ly::QT_TIER;
          const float2 *lp = lpol + lut_off(ti), *la = laz + lut_off(ti);
          const uint8_t *ra = qa ? xst[1] : xst[0], *rb = qb ? xst[1] : xst[0];
          switch (bits) {
            case 4: ada_2page_f4<G, Ly::QT_HALF, 8>(ra, rb, q0, smem_u32(lp), smem_u32(la), lane, fa, fb); break;
            case 3: ada_2page_gen<3, G, Ly::QT_HALF>(ra, rb, q0, lp, la, lane, fa, fb); break;
            case 6: ada_2page_gen<6, G, Ly::QT_HALF>(ra, rb, q0, lp, la, lane, fa, fb); break;
            default: ada_2page_gen<8, G, Ly::QT_HALF>(ra, rb, q0, lp, la, lane, fa, fb); break;
          }
          const float rda = fast_exp2(fmaf((float)ra[256 * bits + (lane & 15)], Dh, Lh));
          const float rdb = fast_exp2(fmaf((float)rb[256 * bits + (lane & 15)], Dh, Lh));
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float va = scg[g] * rda * fa[g], vb = scg[g] * rdb * fb[g];
            if (qa == 0) l2[0][g] = va;
            else l2[1][g] = va;
            if (qb == 1) l2[1][g] = vb;
          }
        }
      } else {
        // narrow ring (b <= 4; the producer admits no wider page) and the
        // dense path: a pair of one tier in one pass, other pages alone
        bool paired = false;
        if constexpr (ADA) paired = use[0] && use[1] && mt[0].bits == mt[1].bits && mt[0].bits <= 4;
        if (paired) {
          if constexpr (ADA) {
            float fa[G], fb[G];
            const int ti = tier_of_bits(mt[0].bits);
            const float *q0 = qt + ti * Ly::QT_TIER;
            const float2 *lp = lpol + lut_off(ti), *la = laz + lut_off(ti);
            if (mt[0].bits == 4)
              ada_2page_f4<G, Ly::QT_HALF, G == 8 ? 4 : 2>(xst[0], xst[1], q0, smem_u32(lp), smem_u32(la), lane, fa,
                                                          fb);
            else
              ada_2page_f<3, G, Ly::QT_HALF>(xst[0], xst[1], q0, lp, la, lane, fa, fb);
            const int bits = mt[0].bits;
            const float ra = fast_exp2(fmaf((float)xst[0][256 * bits + (lane & 15)], Dh, Lh));
            const float rb = fast_exp2(fmaf((float)xst[1][256 * bits + (lane & 15)], Dh, Lh));
#pragma unroll
            for (int g = 0; g < G; ++g) {
              l2[0][g] = scg[g] * ra * fa[g];
              l2[1][g] = scg[g] * rb * fb[g];
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            if (use[q]) page_logits(mt[q], xst[q], l2[q]);  // warp-uniform
          }
        }
      }
      // test the next pair's stages now (their previous phases were this
      // warp's own, so the test is exact); the answer is used after P.V
      {
        const int kn = 2 * (i + NCW);
#pragma unroll
        for (int q = 0; q < 2; ++q)
          ready[q] = kn + q < ke && mbar_test_wait(&full[(kn + q) % NST], (uint32_t)((kn + q) / NST) & 1u);
      }
      // the ring stages are free once the logits are known
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[ka % NST]);
        if (n == 2) mbar_arrive(&empty[(ka + 1) % NST]);
      }
      if (vload) {
        if (!mbar_wait_bounded(vbar, vphase, abort_flag, p.err)) vpending = (int)vphase;
        vphase ^= 1u;
      }
      softmax_pv(use, mt, l2, vslot);
      __syncwarp();
    }

    // ---- this warp's partial of the segment, straight to the workspace
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], o);
    }
    if constexpr (kPackPV) {  // fold the lo columns onto the hi columns
#pragma unroll
      for (int mb = 0; mb < 8; ++mb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (G == 4) d[mb][e] += __shfl_xor_sync(0xffffffffu, d[mb][e], 2);
          else if constexpr (G == 2) d[mb][e] += __shfl_xor_sync(0xffffffffu, d[mb][e], 1);
          else if (e == 0 || e == 2) d[mb][e] += d[mb][e + 1];
        }
      }
    }
    float *part = p.ws + ((int64_t)(c + bh) * NCW + wid) * G * kPartial;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (lane == 0) *reinterpret_cast<float2 *>(part + g * kPartial) = make_float2(m[g], lsum[g]);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int g = 2 * tig + j;
      if (g < G) {
        float *pg = part + g * kPartial + 4;
#pragma unroll
        for (int mb = 0; mb < 8; ++mb) {
          pg[16 * mb + grp] = d[mb][j];
          pg[16 * mb + grp + 8] = d[mb][2 + j];
        }
      }
    }
    // publish the partial: every lane's stores, then one count on the row
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(p.row_done + bh, 1u);
    u = seg_end;
  }
  // After an abort a value load of this warp may still be landing in its
  // slots: wait for it (bounded) before the shared memory is released.
  if (lane == 0 && vpending >= 0) {
    volatile int dummy = 0;
    mbar_wait_bounded(vbar, (uint32_t)vpending, &dummy, nullptr);
  }
}

// ------------------------------------------------------------ merge kernel
// One block per (sequence, query head): combine the partials of every
// (split, consumer warp) that covered the head's kv row.
//   out = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s   (0 when nothing
// was retained).  Launched as a programmatic dependent of the split kernel:
// a block starts on an SM the split grid has left and waits (bounded) until
// the row's count of written partials reaches NCW per covering split, so the
// rows that finish early are merged while the last splits still run.
// partial_out (optional): instead of out, the row's own partial record
// (M, L, 0, 0, o[128]) with o = out, L = sum_s 2^(m_s - M) l_s, for a later
// merge across shards of the sequences' pages (spkv_merge_partials).
constexpr int kMergeThreads = 256;  // 8 warps per (sequence, query head)
template <int G>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const float *ws, const uint32_t *row_done, int C,
                                                              int NCW, const int32_t *ctx_lens, int B, int Hkv,
                                                              int Hq, int max_ctx, int max_pages, void *out,
                                                              int out_bf16, uint32_t *err, float *partial_out) {
  constexpr int kWarps = kMergeThreads / 32, kChunk = kMergeThreads, kBatch = 8;
  __shared__ float wgt[kChunk];
  __shared__ float lsh[kChunk];
  __shared__ int64_t off[kChunk];
  __shared__ float mred[kWarps];
  __shared__ uint32_t nred[kWarps];
  __shared__ __align__(16) float accw[kWarps][kD];
  __shared__ float denw[kWarps];
  const int hq = blockIdx.x % Hq, b = blockIdx.x / Hq;
  const int h = hq / G, g = hq % G, bh = b * Hkv + h;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  __shared__ int32_t Psh[kMaxB + 1];
  __shared__ int32_t pscr[kWarps + 1];
  build_prefix(ctx_lens, B, Hkv, max_ctx, max_pages, nullptr, Psh, pscr, tid, kMergeThreads);
  const Partition part(Psh, B, Hkv, C);
  const int np = (Psh[b + 1] - Psh[b]) / Hkv;
  // lane l of every warp accumulates dims 4 l .. 4 l + 3 over the warp's share
  // of the partials; the warps' sums are added at the end
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f, Mrow = kNegInf;
  if (np > 0) {
    const int64_t a = (int64_t)Psh[b] + (int64_t)h * np, e = a + np;
    const int64_t cf = part.split_of(a, bh), cl = part.split_of(e - 1, bh);
    // splits that hold units of the row (every split in [cf, cl] but empty ones)
    uint32_t live = 0;
    for (int64_t cc = cf + tid; cc <= cl; cc += kMergeThreads)
      live += part.live_in_row(cc, cf, cl) ? 1u : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) live += __shfl_xor_sync(0xffffffffu, live, o);
    if (lane == 0) nred[wid] = live;
    __syncthreads();
    uint32_t nlive = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) nlive += nred[w];
    const uint32_t expected = nlive * (uint32_t)NCW;
    if (tid == 0) {
      const uint64_t t0 = globaltimer_ns();
      uint32_t seen;
      for (;;) {
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(row_done + bh) : "memory");
        if (seen >= expected) break;
        if (globaltimer_ns() - t0 > 1000000000ull) {
          set_err(err, SPKV_DEVERR_TIMEOUT);
          break;
        }
        __nanosleep(256);
      }
    }
    __syncthreads();
    const int64_t nparts = (cl - cf + 1) * NCW;
    float M = kNegInf;
    // pass 1: the max over all partials
    for (int64_t base = 0; base < nparts; base += kMergeThreads) {
      float mm = kNegInf;
      if (base + tid < nparts) {
        const int64_t cc = cf + (base + tid) / NCW;
        const int w = (int)((base + tid) % NCW);
        if (part.live_in_row(cc, cf, cl))
          mm = __ldcg(ws + (((cc + bh) * NCW + w) * G + g) * kPartial);
      }
      M = fmaxf(M, mm);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) mred[wid] = M;
    __syncthreads();
    M = mred[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) M = fmaxf(M, mred[w]);
    Mrow = M;
    if (M != kNegInf) {
      for (int64_t base = 0; base < nparts; base += kChunk) {
        {  // the chunk's weights 2^(m - M), sums l and record offsets (-1: no weight)
          const int i = tid;
          float wv = 0.f, lv = 0.f;
          int64_t o = -1;
          if (base + i < nparts) {
            const int64_t cc = cf + (base + i) / NCW;
            const int w = (int)((base + i) % NCW);
            if (part.live_in_row(cc, cf, cl)) {
              o = (((cc + bh) * NCW + w) * G + g) * kPartial;
              const float2 ml = __ldcg(reinterpret_cast<const float2 *>(ws + o));
              if (ml.x != kNegInf) {
                wv = fast_exp2(ml.x - M);
                lv = ml.y;
              } else {
                o = -1;
              }
            }
          }
          wgt[i] = wv;
          lsh[i] = lv;
          off[i] = o;
        }
        __syncthreads();
        const int n = (int)min((int64_t)kChunk, nparts - base);
        // warp w takes partials w, w + 8, ...; kBatch loads in flight per lane
        for (int i0 = wid; i0 < n; i0 += kWarps * kBatch) {
          float4 v[kBatch];
          float wv[kBatch];
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            const int i = i0 + k * kWarps;
            const int64_t o = i < n ? off[i] : -1;
            wv[k] = 0.f;
            v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (o >= 0) {
              wv[k] = wgt[i];
              den = fmaf(wv[k], lsh[i], den);
              v[k] = __ldcg(reinterpret_cast<const float4 *>(ws + o + 4) + lane);
            }
          }
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            acc.x = fmaf(wv[k], v[k].x, acc.x);
            acc.y = fmaf(wv[k], v[k].y, acc.y);
            acc.z = fmaf(wv[k], v[k].z, acc.z);
            acc.w = fmaf(wv[k], v[k].w, acc.w);
          }
        }
        __syncthreads();
      }
    }
  }
  reinterpret_cast<float4 *>(accw[wid])[lane] = acc;
  if (lane == 0) denw[wid] = den;
  __syncthreads();
  if (tid >= kD) return;
  float num = 0.f, dsum = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    num += accw[w][tid];
    dsum += denw[w];
  }
  const float res = dsum > 0.f ? num / dsum : 0.f;
  if (partial_out) {
    float *pr = partial_out + ((int64_t)b * Hq + hq) * kPartial;
    pr[4 + tid] = res;
    if (tid == 0) *reinterpret_cast<float4 *>(pr) = make_float4(dsum > 0.f ? Mrow : kNegInf, dsum, 0.f, 0.f);
    return;
  }
  const int64_t o = ((int64_t)b * Hq + hq) * kD + tid;
  if (out_bf16) reinterpret_cast<__nv_bfloat16 *>(out)[o] = __float2bfloat16_rn(res);
  else reinterpret_cast<float *>(out)[o] = res;
}

// ------------------------------------------------------- shard merge kernel
// One block per (sequence, query head): out = sum_r w_r o_r / sum_r w_r with
// w_r = 2^(M_r - M) L_r over the R partial records (M_r = -inf: no weight);
// 0 when no shard retained anything.
__global__ void __launch_bounds__(128) merge_partials_kernel(const float *partials, int R, int BH, void *out,
                                                             int out_bf16) {
  const int row = blockIdx.x, tid = threadIdx.x;
  float M = kNegInf;
  for (int r = 0; r < R; ++r) M = fmaxf(M, partials[((int64_t)r * BH + row) * kPartial]);
  float num = 0.f, den = 0.f;
  if (M != kNegInf) {
    for (int r = 0; r < R; ++r) {
      const float *pr = partials + ((int64_t)r * BH + row) * kPartial;
      const float2 ml = *reinterpret_cast<const float2 *>(pr);
      if (ml.x == kNegInf) continue;
      const float w = fast_exp2(ml.x - M) * ml.y;
      num = fmaf(w, pr[4 + tid], num);
      den += w;
    }
  }
  const float res = den > 0.f ? num / den : 0.f;
  const int64_t o = (int64_t)row * kD + tid;
  if (out_bf16) reinterpret_cast<__nv_bfloat16 *>(out)[o] = __float2bfloat16_rn(res);
  else reinterpret_cast<float *>(out)[o] = res;
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
  __shared__ double pol_c2[kLutEntries], az_c2[kLutEntries];
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
  build_edge_tables(pol_c2, az_c2, lane, 32);
  for (uint32_t i = lane * 16; i < rsz; i += 32 * 16)
    *reinterpret_cast<uint4 *>(rec + i) = *reinterpret_cast<const uint4 *>(p.arena + roff + i);
  __syncwarp();
  for (int g = 0; g < G; ++g) {
    const float n = ada_qprep_row<G, QT_HALF>(p.q + ((int64_t)b * p.Hq + (int64_t)h * G + g) * kD, g, lpol, laz,
                                              pol_c2, az_c2, qt, lane, 0xfu,
                                              (p.flags & SPKV_DECODE_EXACT_Q) != 0u);
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
template <bool ADA, int G, bool NW>
int blocks_per_sm(size_t smem) {
  static int configured[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(split_kernel<ADA, G, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Layout<ADA, G, NW>::bytes(kMaxB)) != cudaSuccess)
      return -1;
    configured[dev] = 1;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, split_kernel<ADA, G, NW>, Layout<ADA, G, NW>::THREADS,
                                                    smem) != cudaSuccess)
    return -1;
  return n;
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
  float *partial_out = nullptr;
};

template <bool ADA, int G, bool NW>
spkv_status launch_g(const DecodeArgs &a, const CUtensorMap &vmap, cudaStream_t stream) {
  using Ly = Layout<ADA, G, NW>;
  const size_t smem = Ly::bytes(a.sp.B);
  if (blocks_per_sm<ADA, G, NW>(smem) < 1) return SPKV_ERR_CUDA;
  // the row counters start at zero in every launch
  if (cudaMemsetAsync(a.sp.row_done, 0, (size_t)a.sp.B * a.sp.Hkv * sizeof(uint32_t), stream) != cudaSuccess)
    return SPKV_ERR_CUDA;
  split_kernel<ADA, G, NW><<<a.num_splits, Ly::THREADS, smem, stream>>>(a.sp, vmap);
  if (cudaGetLastError() != cudaSuccess) return SPKV_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.sp.B * a.sp.Hq));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float *ws = a.sp.ws;
  const uint32_t *done = a.sp.row_done;
  if (cudaLaunchKernelEx(&cfg, merge_kernel<G>, ws, done, a.num_splits, Ly::NCW, a.sp.ctx_lens, a.sp.B, a.sp.Hkv,
                         a.sp.Hq, a.sp.max_ctx, a.sp.max_pages, a.out, a.out_bf16, a.sp.err,
                         a.partial_out) != cudaSuccess)
    return SPKV_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}

template <bool ADA, bool NW>
spkv_status launch_nw(const DecodeArgs &a, const CUtensorMap &vmap, cudaStream_t stream) {
  switch (a.G) {
    case 1: return launch_g<ADA, 1, NW>(a, vmap, stream);
    case 2: return launch_g<ADA, 2, NW>(a, vmap, stream);
    case 4: return launch_g<ADA, 4, NW>(a, vmap, stream);
    case 8: return launch_g<ADA, 8, NW>(a, vmap, stream);
  }
  return SPKV_ERR_UNSUPPORTED;
}

// Split + merge launches.  An ADA cache whose pages are all b <= 4 (tier
// mask within {3, 4}) runs the narrow-stage kernel.
template <bool ADA>
spkv_status launch_split_and_merge(const DecodeArgs &a, cudaStream_t stream) {
  CUtensorMap vmap;
  if (!make_value_tensor_map(&vmap, a.sp.v_pages, (uint64_t)a.sp.num_pages * a.sp.Hkv * kPage))
    return a.sp.num_pages == 0 ? SPKV_ERR_INVALID_ARG : SPKV_ERR_CUDA;
  if constexpr (ADA) {
    if ((a.sp.tiers & ~0x3u) == 0u) return launch_nw<true, true>(a, vmap, stream);
  }
  return launch_nw<ADA, false>(a, vmap, stream);
}

size_t ws_partials_bytes(int B, int Hq, int Hkv, int C) {
  return ((size_t)(C + B * Hkv) * kNCWMax * (size_t)(Hq / Hkv) * kPartial * sizeof(float) + 15) / 16 * 16;
}
size_t ws_bytes_for(int B, int Hq, int Hkv, int C) {
  return ws_partials_bytes(B, Hq, Hkv, C) + ((size_t)B * Hkv * sizeof(uint32_t) + 15) / 16 * 16;
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
  sp.row_done = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(ws) + ws_partials_bytes(B, Hq, Hkv, C));
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
  sp.tiers = c->tiers ? c->tiers : 0xfu;
  sp.flags = 0u;
  sp.new_k = nullptr;
  sp.new_v = nullptr;
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

namespace spkv {
namespace {
spkv_status decode_ada(const spkv_cache *cache, const uint16_t *new_k, const uint16_t *new_v, const uint16_t *q,
                       int32_t B, int32_t Hq, const int32_t *block_table, int32_t max_pages, const int32_t *ctx_lens,
                       int32_t max_ctx, void *out, int32_t out_is_bf16, void *ws, size_t ws_bytes,
                       int32_t num_splits, uint32_t flags, void *stream, float *partial_out = nullptr) {
  if (flags & ~SPKV_DECODE_EXACT_Q) return SPKV_ERR_INVALID_ARG;
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  DecodeArgs a;
  fill_cache(a.sp, cache);
  a.sp.flags = flags;
  a.sp.new_k = new_k;
  a.sp.new_v = new_v;
  st = prep_batch(a.sp, cache->num_kv_heads, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, out, ws, ws_bytes,
                  num_splits, &a.G, &a.num_splits);
  if (st != SPKV_OK) return st;
  if (B == 0) return SPKV_OK;
  a.out = out;
  a.out_bf16 = out_is_bf16 ? 1 : 0;
  a.partial_out = partial_out;
  return launch_split_and_merge<true>(a, (cudaStream_t)stream);
}
}  // namespace
}  // namespace spkv

extern "C" spkv_status spkv_decode_attention_partial(const spkv_cache *cache, const uint16_t *q, int32_t B,
                                                     int32_t Hq, const int32_t *block_table, int32_t max_pages,
                                                     const int32_t *ctx_lens, int32_t max_ctx, float *partial_out,
                                                     void *ws, size_t ws_bytes, int32_t num_splits, uint32_t flags,
                                                     void *stream) {
  if (B > 0 && (!partial_out || ((uintptr_t)partial_out & 15))) return SPKV_ERR_INVALID_ARG;
  // out is unused on this path; prep_batch only needs an aligned non-null pointer
  return decode_ada(cache, nullptr, nullptr, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, partial_out, 0,
                    ws, ws_bytes, num_splits, flags, stream, partial_out);
}

extern "C" spkv_status spkv_merge_partials(const float *partials, int32_t R, int32_t B, int32_t Hq, void *out,
                                           int32_t out_is_bf16, void *stream) {
  if (R < 1 || B < 0 || Hq < 1) return SPKV_ERR_INVALID_ARG;
  if (B == 0) return SPKV_OK;
  if (!partials || !out || ((uintptr_t)partials & 15) || ((uintptr_t)out & 15)) return SPKV_ERR_INVALID_ARG;
  if ((int64_t)B * Hq > 0x7fffffff) return SPKV_ERR_UNSUPPORTED;
  merge_partials_kernel<<<B * Hq, 128, 0, (cudaStream_t)stream>>>(partials, R, B * Hq, out, out_is_bf16 ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}

extern "C" spkv_status spkv_decode_attention_ex(const spkv_cache *cache, const uint16_t *q, int32_t B, int32_t Hq,
                                                const int32_t *block_table, int32_t max_pages,
                                                const int32_t *ctx_lens, int32_t max_ctx, void *out,
                                                int32_t out_is_bf16, void *ws, size_t ws_bytes, int32_t num_splits,
                                                uint32_t flags, void *stream) {
  return decode_ada(cache, nullptr, nullptr, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, out, out_is_bf16,
                    ws, ws_bytes, num_splits, flags, stream);
}

extern "C" spkv_status spkv_decode_attention_append(const spkv_cache *cache, const uint16_t *new_keys,
                                                    const uint16_t *new_values, const uint16_t *q, int32_t B,
                                                    int32_t Hq, const int32_t *block_table, int32_t max_pages,
                                                    const int32_t *ctx_lens, int32_t max_ctx, void *out,
                                                    int32_t out_is_bf16, void *ws, size_t ws_bytes,
                                                    int32_t num_splits, uint32_t flags, void *stream) {
  if (B > 0 && (!new_keys || !new_values)) return SPKV_ERR_INVALID_ARG;
  if (((uintptr_t)new_keys & 7) || ((uintptr_t)new_values & 7)) return SPKV_ERR_INVALID_ARG;
  return decode_ada(cache, new_keys, new_values, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, out,
                    out_is_bf16, ws, ws_bytes, num_splits, flags, stream);
}

extern "C" spkv_status spkv_decode_attention(const spkv_cache *cache, const uint16_t *q, int32_t B, int32_t Hq,
                                             const int32_t *block_table, int32_t max_pages,
                                             const int32_t *ctx_lens, int32_t max_ctx, void *out,
                                             int32_t out_is_bf16, void *ws, size_t ws_bytes, int32_t num_splits,
                                             void *stream) {
  return spkv_decode_attention_ex(cache, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, out, out_is_bf16, ws,
                                  ws_bytes, num_splits, 0u, stream);
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

extern "C" spkv_status spkv_debug_logits_ex(const spkv_cache *cache, const uint16_t *q, int32_t B, int32_t Hq,
                                            const int32_t *block_table, int32_t max_pages, const int32_t *ctx_lens,
                                            int32_t max_ctx, float *logits, uint32_t flags, void *stream) {
  if (flags & ~SPKV_DECODE_EXACT_Q) return SPKV_ERR_INVALID_ARG;
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  if (B < 0 || Hq < 1 || max_pages < 0 || max_ctx < 0 || Hq % cache->num_kv_heads) return SPKV_ERR_INVALID_ARG;
  const int G = Hq / cache->num_kv_heads;
  if (!g_supported(G)) return SPKV_ERR_UNSUPPORTED;
  if (B == 0 || max_ctx == 0) return SPKV_OK;
  if (!q || !block_table || !ctx_lens || !logits || ((uintptr_t)q & 7)) return SPKV_ERR_INVALID_ARG;
  SplitParams sp;
  fill_cache(sp, cache);
  sp.flags = flags;
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

extern "C" spkv_status spkv_debug_logits(const spkv_cache *cache, const uint16_t *q, int32_t B, int32_t Hq,
                                         const int32_t *block_table, int32_t max_pages, const int32_t *ctx_lens,
                                         int32_t max_ctx, float *logits, void *stream) {
  return spkv_debug_logits_ex(cache, q, B, Hq, block_table, max_pages, ctx_lens, max_ctx, logits, 0u, stream);
}
