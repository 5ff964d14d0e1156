// spkv_encode.cuh -- a key into its page slot: one thread per key for the
// bulk encode kernel (spkv_encode_keys), one warp per key for small calls and
// the decode kernel's fused single-token append (spkv_decode_attention_append);
// the two forms make the same decisions with the same roundings, so they write
// the same bytes for a key.
//
// Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
// for Efficient Long-Context Inference", technical summary section 2.1
// (r = ||k||, phi = Phi(k^); quantised radius and packed angle codes).  Every
// angle code is decided in fp64 from the exact squares of the bf16 inputs;
// the radius code uses fp64 log2.
//
// Order of the suffix sums S_i = sum_{j >= i} x_j^2 (fixed, so that every
// path that encodes a key rounds them alike): the key is cut into 32 groups of
// four dims; group g's local sums are s3 = x3^2, s2 = fma(x2, x2, s3),
// s1 = fma(x1, x1, s2), s0 = fma(x0, x0, s1) (x_k = dim 4g + k); T_32 = 0 and
// T_g = s0 + T_(g+1); then S_(4g+k) = s_k + T_(g+1).
#pragma once

#include "spkv_common.cuh"

namespace spkv {

// The same codes as polar_code, by a search over half the edges: with
// S > 0, the sign of x fixes the half of [0, pi] the angle lies in --
//   x > 0: the code is the largest k in [0, 2^(b-1)) with x^2 <= S c2[k]
//          (k = 0 always: c2[0] = 1, x^2 <= S);
//   x < 0: the code is 2^(b-1) + the largest j in [0, 2^(b-1)) with j = 0 or
//          x^2 >= S c2[2^(b-1) + j], tested as -x^2 <= S (-c2[2^(b-1) + j])
//          (negation is exact, so this is the same test);
//   x = 0: the angle is pi/2 exactly, code 2^(b-1) -- the x < 0 branch gives
//          it: -0 <= -S c2[2^(b-1) + j] fails for every j >= 1 (c2 > 0
//          there, and S c2 >= 2^-280 for bf16 inputs, so it never rounds to 0)
// (polar_reaches' tests, in which "x <= 0" and "x < 0" are fixed per angle;
// c2[2^(b-1)] = 0 exactly, so k = 2^(b-1) is not reached for x > 0).  The
// test is monotone (true up to the code, false above), so the search adds the
// steps 2^(b-2), ..., 1 to the code while the test holds, starting from 0
// (x > 0) or 2^(b-1) (x <= 0): one fp64 product and one comparison per step,
// sx2 <= S e[k] with sx2 = x |x| (exactly x^2 or -x^2).
//   HS (half-signed table, build_edge_tables(..., true)): e[k] = c2[k] below
//       2^(b-1) and -c2[k] from 2^(b-1) on;
//   !HS (the plain table): e[k] = c2[k], and the sign goes on S instead,
//       sx2 <= (-S) c2[k] for x <= 0 (the same products, negated exactly).
// An fp64 load from a 32-bit shared-window address (the edge tables are
// written before the barrier that precedes every search).
__device__ __forceinline__ double lds_f64(uint32_t addr) {
  double v;
  asm volatile("ld.shared.f64 %0, [%1];" : "=d"(v) : "r"(addr));
  return v;
}

template <int BITS, bool HS = false>
__device__ __forceinline__ int polar_code_half(double x, double S, const double *c2) {
  constexpr int H = 1 << (BITS - 1);
  const bool pos = x > 0.0;
  const double sx2 = x * fabs(x);
  const double sS = HS || pos ? S : -S;
  const uint32_t base = smem_u32(c2);
  uint32_t a = pos ? base : base + 8u * H;  // the entry of the code so far
#pragma unroll
  for (int step = H / 2; step >= 1; step >>= 1) {
    const uint32_t an = a + 8u * step;
    a = sx2 <= sS * lds_f64(an) ? an : a;
  }
  return S == 0.0 ? 0 : (int)((a - base) >> 3);
}

// Non-uniform quantiser (an f_b variant): polar angle a has its own edges,
// ec[j - 1] = cos theta_j (j = 1 .. 2^b - 1, increasing angles), and its code
// is the largest j whose edge it reaches (j = 0 always), by the same exact
// test: phi >= theta <=> x <= sqrt(S) cos theta.  With signed squares it is
// one comparison for either sign of cos theta:
//   x |x| <= S (c |c|)   (c = cos theta)
// -- for c >= 0 it holds iff x <= 0 or x^2 <= S c^2, for c < 0 iff x < 0 and
// x^2 >= S c^2 (S c^2 > 0 there), which is the test; c |c| and x |x| are the
// rounded squares with a sign, so the products round as S (c c) does.  The
// search adds the steps 2^(b-1), ..., 1 while the test holds.
template <int BITS>
__device__ __forceinline__ int polar_code_nu(double x, double S, const double *ec) {
  const double sx2 = x * fabs(x);
  int k = 0;
#pragma unroll
  for (int step = 1 << (BITS - 1); step >= 1; step >>= 1) {
    const double c = ec[k + step - 1];
    k = sx2 <= S * (c * fabs(c)) ? k + step : k;
  }
  return S == 0.0 ? 0 : k;
}

// The slot's bitstream (codes LSB first, code i at bits [i b, i b + b)) is
// built from the top group of four codes down in a 64-bit accumulator
// (acc = acc << 4 b | grp, grp holding field i + k at bits [k b, k b + b)),
// and word w = bits [32 w, 32 w + 32) is taken once the lowest code added
// starts at or below bit 32 w (4 b <= 32: at most one word per group, and at
// most 32 + 4 b <= 64 bits pending); the four words of chunk c = w / 4 go out
// as one 16-byte store at recp + (16 c + slot) 16 (chunk-major record layout).
struct SlotWords {
  uint64_t acc = 0u;
  int w;       // next word to take (descending)
  uint4 stage;  // the chunk being filled
  uint8_t *recp;
  int slot;
  __device__ __forceinline__ SlotWords(uint8_t *r, int s, int nwords) : w(nwords - 1), recp(r), slot(s) {
    stage = make_uint4(0u, 0u, 0u, 0u);
  }
  template <int BITS>
  __device__ __forceinline__ void push_group(int i, uint32_t grp) {
    acc = (acc << (4 * BITS)) | grp;
    if (i * BITS <= 32 * w) {  // word w complete
      const uint32_t word = (uint32_t)(acc >> (32 * w - i * BITS));
      const int wic = w & 3;
      stage.x = wic == 0 ? word : stage.x;
      stage.y = wic == 1 ? word : stage.y;
      stage.z = wic == 2 ? word : stage.z;
      stage.w = wic == 3 ? word : stage.w;
      if (wic == 0) *reinterpret_cast<uint4 *>(recp + ((w >> 2) * 16 + slot) * 16) = stage;
      --w;
    }
  }
};

// Four dims of a key (bf16 bits) as fp64.
__device__ __forceinline__ void bf16x4_to_f64(uint2 raw, double (&x)[4]) {
  x[0] = bf16_to_f64(raw.x & 0xffffu);
  x[1] = bf16_to_f64(raw.x >> 16);
  x[2] = bf16_to_f64(raw.y & 0xffffu);
  x[3] = bf16_to_f64(raw.y >> 16);
}

// The calling thread encodes key[0..127] (bf16 bits, 8-byte aligned) into
// slot `slot` of the (page, kv head) record at recp, whose pages have bit
// width BITS: the 127 angle codes, packed LSB first into the slot's
// chunk-major bitstream, and the radius byte after the 256 b code bytes.
// pc2 / ac2: this tier's fp64 cos^2 edge tables (build_edge_tables).
// NU: the non-uniform quantiser's polar codes, against nu_ec (row a: the
// 2^b - 1 edge cosines of angle a); the azimuth and radius are unchanged.
template <int BITS, bool NU = false>
__device__ __forceinline__ void encode_key_lane(const uint16_t *key, uint8_t *recp, int slot, float Lf, float Df,
                                                const double *pc2, const double *ac2, uint32_t *err,
                                                const double *nu_ec = nullptr) {
  constexpr int NE = (1 << BITS) - 1;
  auto polar = [&](int a, double x, double S) -> uint32_t {
    if constexpr (NU) return (uint32_t)polar_code_nu<BITS>(x, S, nu_ec + a * NE);
    else return (uint32_t)polar_code_half<BITS, true>(x, S, pc2);
  };
  SlotWords sw(recp, slot, 4 * BITS);
  const uint2 *kr = reinterpret_cast<const uint2 *>(key);
  // ---- group 31: dims 124..127 (angles 124, 125 polar, 126 the azimuth, 127 padding)
  double x[4], s[4];
  bf16x4_to_f64(kr[31], x);
  s[3] = x[3] * x[3];
  s[2] = fma(x[2], x[2], s[3]);
  s[1] = fma(x[1], x[1], s[2]);
  s[0] = fma(x[0], x[0], s[1]);
  double T = s[0] + 0.0;  // T_31 (T_32 = 0)
  sw.push_group<BITS>(124, polar(124, x[0], s[0] + 0.0) | polar(125, x[1], s[1] + 0.0) << BITS |
                               (uint32_t)azimuth_code<BITS>(x[2], x[3], s[2] + 0.0, ac2) << (2 * BITS));
  // (field 127, the padding, is 0)
  // ---- groups 30 .. 0; each group's dims are loaded two groups ahead,
  // through a shift register
  uint2 pf[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) pf[j] = kr[30 - j];
#pragma unroll 1
  for (int g = 30; g >= 0; --g) {
    bf16x4_to_f64(pf[0], x);
    pf[0] = pf[1];
    pf[1] = g >= 2 ? kr[g - 2] : make_uint2(0u, 0u);
    s[3] = x[3] * x[3];
    s[2] = fma(x[2], x[2], s[3]);
    s[1] = fma(x[1], x[1], s[2]);
    s[0] = fma(x[0], x[0], s[1]);
    const double Tn = T;  // T_(g+1)
    T = s[0] + Tn;        // T_g
    uint32_t grp = 0u;
#pragma unroll
    for (int k = 3; k >= 0; --k) grp |= polar(4 * g + k, x[k], s[k] + Tn) << (k * BITS);
    sw.push_group<BITS>(4 * g, grp);
  }
  // ---- radius code from S_0 = T_0 = ||k||^2
  int c = 0;
  if (!(Df > 0.0f) || !isfinite(Df) || !isfinite(Lf)) {
    set_err(err, SPKV_DEVERR_RADIUS);
  } else if (T > 0.0) {
    const double tr = (log2(sqrt(T)) - (double)Lf) / (double)Df + 0.5;
    c = tr <= 0.0 ? 0 : tr >= 255.0 ? 255 : (int)floor(tr);
  }
  recp[256 * BITS + slot] = (uint8_t)c;
}

// encode_key_lane for the tier of `bits` (a valid tier: 3, 4, 6 or 8).
__device__ __forceinline__ void encode_key_lane_bits(int bits, const uint16_t *key, uint8_t *recp, int slot,
                                                     float Lf, float Df, const double *pol_c2,
                                                     const double *az_c2, uint32_t *err) {
  const int t = tier_of_bits(bits);
  const double *pc2 = pol_c2 + lut_off(t), *ac2 = az_c2 + lut_off(t);
  switch (bits) {
    case 3: encode_key_lane<3>(key, recp, slot, Lf, Df, pc2, ac2, err); break;
    case 4: encode_key_lane<4>(key, recp, slot, Lf, Df, pc2, ac2, err); break;
    case 6: encode_key_lane<6>(key, recp, slot, Lf, Df, pc2, ac2, err); break;
    default: encode_key_lane<8>(key, recp, slot, Lf, Df, pc2, ac2, err); break;
  }
}

// encode_key_lane with the non-uniform polar codes, for b = bits (a valid
// tier); nu_ec: the 126 x (2^b - 1) edge cosines of the polar angles.
__device__ __forceinline__ void encode_key_lane_nu_bits(int bits, const uint16_t *key, uint8_t *recp, int slot,
                                                        float Lf, float Df, const double *az_c2,
                                                        const double *nu_ec, uint32_t *err) {
  const double *ac2 = az_c2 + lut_off(tier_of_bits(bits));
  switch (bits) {
    case 3: encode_key_lane<3, true>(key, recp, slot, Lf, Df, nullptr, ac2, err, nu_ec); break;
    case 4: encode_key_lane<4, true>(key, recp, slot, Lf, Df, nullptr, ac2, err, nu_ec); break;
    case 6: encode_key_lane<6, true>(key, recp, slot, Lf, Df, nullptr, ac2, err, nu_ec); break;
    default: encode_key_lane<8, true>(key, recp, slot, Lf, Df, nullptr, ac2, err, nu_ec); break;
  }
}

// The same bytes as encode_key_lane, computed by a whole warp (the fused
// append's form, one key at a time): lane l holds dims 4l .. 4l+3 (group l)
// and forms the group's local sums; the group suffix T_l = s0_l + T_(l+1)
// runs down the lanes one addition at a time (the same additions, so the
// same roundings); each lane decides its four codes, and the slot's words are
// put together by funnel shifts across lanes.
template <int BITS, bool HS>
__device__ __forceinline__ void encode_key_warp_seq(const uint16_t *key, uint8_t *recp, int slot, float Lf,
                                                    float Df, const double *pc2, const double *ac2, int lane,
                                                    uint32_t *err) {
  double x[4], s[4];
  bf16x4_to_f64(*reinterpret_cast<const uint2 *>(key + 4 * lane), x);
  s[3] = x[3] * x[3];
  s[2] = fma(x[2], x[2], s[3]);
  s[1] = fma(x[1], x[1], s[2]);
  s[0] = fma(x[0], x[0], s[1]);
  double T = 0.0;  // lane l: T_l once the chain has passed it
  if (lane == 31) T = s[0] + 0.0;
#pragma unroll 1
  for (int l = 30; l >= 0; --l) {
    const double up = __shfl_sync(0xffffffffu, T, l + 1);
    if (lane == l) T = s[0] + up;
  }
  double Tn = __shfl_down_sync(0xffffffffu, T, 1);  // T_(l+1)
  if (lane == 31) Tn = 0.0;
  uint32_t grp = 0u;  // this lane's four codes, LSB first
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int a = 4 * lane + k;
    const double S = s[k] + Tn;
    int c = polar_code_half<BITS, HS>(x[k], S, pc2);
    if (a >= 126) c = a == 126 ? azimuth_code<BITS>(x[2], x[3], S, ac2) : 0;
    grp |= (uint32_t)c << (k * BITS);
  }
  // word w = bits [32 w, 32 w + 32): from the groups of lanes first ..
  // first + SPAN - 1, first = 32 w / (4 b)
  constexpr int GB = 4 * BITS, SPAN = BITS == 3 ? 4 : (BITS == 8 ? 1 : 2);
  const int first = (32 * lane) / GB, off = 32 * lane - first * GB;
  uint64_t acc = 0u;
#pragma unroll
  for (int j = 0; j < SPAN; ++j) {
    const uint32_t gj = __shfl_sync(0xffffffffu, grp, min(first + j, 31));
    acc |= (uint64_t)gj << (j * GB);
  }
  if (lane < GB) {
    const int chunk = lane >> 2, wic = lane & 3;
    *reinterpret_cast<uint32_t *>(recp + (chunk * 16 + slot) * 16 + wic * 4) = (uint32_t)(acc >> off);
  }
  // ---- radius code from S_0 = T_0 (lane 0)
  if (lane == 0) {
    int c = 0;
    if (!(Df > 0.0f) || !isfinite(Df) || !isfinite(Lf)) {
      set_err(err, SPKV_DEVERR_RADIUS);
    } else if (T > 0.0) {
      const double tr = (log2(sqrt(T)) - (double)Lf) / (double)Df + 0.5;
      c = tr <= 0.0 ? 0 : tr >= 255.0 ? 255 : (int)floor(tr);
    }
    recp[256 * BITS + slot] = (uint8_t)c;
  }
  __syncwarp();
}

// encode_key_warp_seq for the tier of `bits` (a valid tier); HS: pol_c2 is
// the half-signed table (build_edge_tables(..., true)).
template <bool HS = false>
__device__ __forceinline__ void encode_key_warp_seq_bits(int bits, const uint16_t *key, uint8_t *recp, int slot,
                                                         float Lf, float Df, const double *pol_c2,
                                                         const double *az_c2, int lane, uint32_t *err) {
  const int t = tier_of_bits(bits);
  const double *pc2 = pol_c2 + lut_off(t), *ac2 = az_c2 + lut_off(t);
  switch (bits) {
    case 3: encode_key_warp_seq<3, HS>(key, recp, slot, Lf, Df, pc2, ac2, lane, err); break;
    case 4: encode_key_warp_seq<4, HS>(key, recp, slot, Lf, Df, pc2, ac2, lane, err); break;
    case 6: encode_key_warp_seq<6, HS>(key, recp, slot, Lf, Df, pc2, ac2, lane, err); break;
    default: encode_key_warp_seq<8, HS>(key, recp, slot, Lf, Df, pc2, ac2, lane, err); break;
  }
}

}  // namespace spkv
