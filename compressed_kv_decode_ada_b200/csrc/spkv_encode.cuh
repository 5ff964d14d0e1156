// spkv_encode.cuh -- one warp encodes one key into its page slot: shared by
// the bulk encode kernel (spkv_encode_keys) and the decode kernel's fused
// single-token append (spkv_decode_attention_append), so both write the same
// bytes for the same key.
//
// Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
// for Efficient Long-Context Inference", technical summary section 2.1
// (r = ||k||, phi = Phi(k^); quantised radius and packed angle codes).  Every
// angle code is decided in fp64 from the exact squares of the bf16 inputs
// (lane_codes); the radius code uses fp64 log2.
#pragma once

#include "spkv_common.cuh"

namespace spkv {

// Word w (32 bits) of a slot's bitstream, from the byte-per-angle codes.
template <int BITS>
__device__ __forceinline__ uint32_t pack_word(const uint8_t *codes, int w) {
  const int lo_bit = 32 * w;
  const int a0 = lo_bit / BITS, a1 = min(127, (lo_bit + 31) / BITS);
  uint32_t v = 0;
  for (int a = a0; a <= a1; ++a) {
    const int sh = a * BITS - lo_bit;
    const uint32_t c = codes[a];
    v |= sh >= 0 ? (c << sh) : (c >> (-sh));
  }
  return v;
}

// The calling warp encodes key[0..127] (bf16 bits; lane l holds dims
// 4l..4l+3) into slot `slot` of the (page, kv head) record at recp, whose
// pages have bit width `bits` (a valid tier): the 127 angle codes, packed
// LSB-first into the slot's chunk-major bitstream, and the radius byte after
// the 256 b code bytes.  codes_smem: 128 bytes of this warp's shared memory.
// pol_c2 / az_c2: the fp64 cos^2 edge tables (build_edge_tables).
__device__ __forceinline__ void encode_key_warp(const uint16_t *key, int bits, uint8_t *recp, int slot, float Lf,
                                                float Df, const double *pol_c2, const double *az_c2,
                                                uint8_t *codes_smem, int lane, uint32_t *err) {
  // ---- x (4 per lane); exact squares and suffix sums in fp64
  const uint2 raw = *reinterpret_cast<const uint2 *>(key + 4 * lane);
  double x[4], S[4];
  lane_suffix_sums(raw, lane, x, S);
  const double x127 = __shfl_sync(0xffffffffu, x[3], 31);

  // ---- angle codes (fp64 decisions), one byte per angle in shared memory
  int c4[4];
  switch (bits) {
    case 3: lane_codes<3>(x, S, x127, lane, pol_c2, az_c2, c4); break;
    case 4: lane_codes<4>(x, S, x127, lane, pol_c2, az_c2, c4); break;
    case 6: lane_codes<6>(x, S, x127, lane, pol_c2, az_c2, c4); break;
    default: lane_codes<8>(x, S, x127, lane, pol_c2, az_c2, c4); break;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) codes_smem[4 * lane + k] = (uint8_t)c4[k];
  __syncwarp();

  // ---- pack: lane w < 4b builds word w; store chunk-major
  if (lane < 4 * bits) {
    uint32_t word;
    switch (bits) {
      case 3: word = pack_word<3>(codes_smem, lane); break;
      case 4: word = pack_word<4>(codes_smem, lane); break;
      case 6: word = pack_word<6>(codes_smem, lane); break;
      default: word = pack_word<8>(codes_smem, lane); break;
    }
    const int chunk = lane >> 2, wic = lane & 3;
    *reinterpret_cast<uint32_t *>(recp + (chunk * 16 + slot) * 16 + wic * 4) = word;
  }
  // ---- radius code (lane 0 holds S_0 = ||k||^2)
  if (lane == 0) {
    int c = 0;
    if (!(Df > 0.0f) || !isfinite(Df) || !isfinite(Lf)) {
      set_err(err, SPKV_DEVERR_RADIUS);
    } else if (S[0] > 0.0) {
      const double t = (log2(sqrt(S[0])) - (double)Lf) / (double)Df + 0.5;
      c = t <= 0.0 ? 0 : t >= 255.0 ? 255 : (int)floor(t);
    }
    recp[256 * bits + slot] = (uint8_t)c;
  }
  __syncwarp();
}

}  // namespace spkv
