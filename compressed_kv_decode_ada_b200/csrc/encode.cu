// encode.cu -- spkv_encode_keys: bf16 keys -> (uint8 log radius code, b-bit
// angle codes) appended to their page slots through the block table.
//
// Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
// for Efficient Long-Context Inference", technical summary section 2.1
// ("spherical parametrisation": r = ||k||, phi = Phi(k^); ADA "stores
// quantised radii and packed angle codes") and 2.3 ("maps dense keys to
// spherical codes ... stores them in a compressed format").
//
// Every code is decided in fp64 without evaluating any angle: the squares of
// bf16 inputs are exact in fp64, and
//   phi_i >= theta_k  <=>  x_i <= sqrt(S_i) cos(theta_k)
// (S_i = sum_{j >= i} x_j^2) is decided from x_i^2 versus S_i cos^2(theta_k)
// plus the signs.  The code is the largest k whose edge theta_k the angle
// reaches (a stepped search over the edges of the half of [0, pi] the sign of
// x_i gives, one product and one comparison per step), i.e.
// floor(phi 2^b / pi) clamped to 2^b - 1 -- ties go to the upper cell.  The
// azimuth (angle 127, range [0, 2 pi)) uses the same test on (x_126, x_127)
// with the half-plane given by the sign of x_127.  The radius code uses fp64
// log2.  One thread encodes one key in bulk calls, one warp per key in small
// ones (spkv_encode.cuh).
#include "spkv_encode.cuh"

namespace spkv {
namespace {

constexpr int kEncThreads = 256;
constexpr int64_t kEncWarpItems = 512;  // up to this many items: a warp per key

struct EncodeParams {
  uint8_t *arena;
  uint64_t arena_bytes;
  const spkv_page_hdr *hdr;
  const float *rad_lo, *rad_step;
  uint16_t *v_pages;
  uint32_t *err;
  int Hkv, num_pages;
  const uint16_t *keys, *values;
  const int32_t *start_pos, *block_table;
  const int32_t *seq_start, *dst_pos;  // scattered placement (start_pos unused)
  int B, n_new, max_pages;
  int64_t items;  // B * n_new * Hkv, or total_tokens * Hkv when scattered
  // non-uniform quantiser (nullptr: the uniform one): every page must have
  // b = nu_bits; nu_ec holds the 126 x (2^b - 1) polar edge cosines
  const double *nu_ec;
  int nu_bits;
};

// Where item (key, kv head) `item` goes: its kv head, page and slot, or the
// device-error bits that rule it out; skip: a packed token with a negative
// position (nothing to write).
struct EncPlace {
  int h, pid, slot;
  uint32_t st;
  bool skip;
};

__device__ __forceinline__ EncPlace enc_place(const EncodeParams &p, int64_t item) {
  EncPlace pl{0, -1, 0, 0u, false};
  int64_t bn;
  if (p.items <= 0x7fffffff) {  // 32-bit division where it fits
    const uint32_t i32 = (uint32_t)item, hk = (uint32_t)p.Hkv, q = i32 / hk;
    pl.h = (int)(i32 - q * hk);
    bn = q;
  } else {
    pl.h = (int)(item % p.Hkv);
    bn = item / p.Hkv;
  }
  int b, pos;
  if (p.dst_pos) {  // token bn of the concatenated sequences, to dst_pos[bn]
    pos = p.dst_pos[bn];
    if (pos < 0) {
      pl.skip = true;
      return pl;
    }
    int lo = 0, hi = p.B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if ((int64_t)p.seq_start[mid] <= bn) lo = mid;
      else hi = mid;
    }
    b = lo;
    if (bn < (int64_t)p.seq_start[b] || bn >= (int64_t)p.seq_start[b + 1]) {
      pl.st = SPKV_DEVERR_CTX;
      return pl;
    }
  } else if (bn <= 0xffffffffLL) {
    const uint32_t nn = (uint32_t)p.n_new, q = (uint32_t)bn / nn;
    b = (int)q;
    pos = p.start_pos[b] + (int)((uint32_t)bn - q * nn);
  } else {
    b = (int)(bn / p.n_new);
    pos = p.start_pos[b] + (int)(bn % p.n_new);
  }
  if (pos < 0 || pos >= p.max_pages * kPage) {
    pl.st = SPKV_DEVERR_CTX;
    return pl;
  }
  pl.slot = pos % kPage;
  pl.pid = p.block_table[(int64_t)b * p.max_pages + pos / kPage];
  if (pl.pid < 0 || pl.pid >= p.num_pages) pl.st = SPKV_DEVERR_PAGE_ID;
  return pl;
}

// Checks of an item's page header: its bit width and record offset, or the
// device-error bits that rule it out.
__device__ __forceinline__ uint32_t enc_record(const EncodeParams &p, const EncPlace &pl, int &bits, uint64_t &rec) {
  if (pl.st) return pl.st;
  const spkv_page_hdr hd = p.hdr[pl.pid];
  bits = hd.bits;
  if (tier_of_bits(bits) < 0) return SPKV_DEVERR_BITS;
  if (p.nu_ec && bits != p.nu_bits) return SPKV_DEVERR_BITS;
  rec = (uint64_t)hd.code_off16 * 16u + (uint64_t)pl.h * rec_bytes(bits);
  if (rec + rec_bytes(bits) > p.arena_bytes) return SPKV_DEVERR_RECORD;
  return 0u;
}

// Bulk encode: each warp takes 32 consecutive items at a time, one per lane.
// The 32 key rows (8 KB, contiguous) come into the warp's shared-memory
// stage with coalesced loads (rows 264 bytes apart, so the lanes' 8-byte
// reads of their own rows fall in different bank pairs); each lane encodes
// its key from there (encode_key_lane, reading two groups ahead); the value
// rows are copied by the whole warp, a row per instruction (coalesced
// 256-byte reads and writes), eight rows in flight.
constexpr int kEncRowStride = 264;  // bytes per staged key row
struct EncodeSmem {
  double pol_c2[kLutEntries];
  double az_c2[kLutEntries];
  alignas(16) uint8_t rows[kEncThreads / 32][32 * kEncRowStride];
};

__global__ void __launch_bounds__(kEncThreads, 3) encode_kernel(const EncodeParams p) {
  extern __shared__ __align__(16) uint8_t enc_smem_raw[];
  EncodeSmem &sm = *reinterpret_cast<EncodeSmem *>(enc_smem_raw);
  build_edge_tables(sm.pol_c2, sm.az_c2, threadIdx.x, kEncThreads, true);
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint8_t *stage = sm.rows[wid];
  const int64_t nbatch = (p.items + 31) / 32;
  const int64_t wstep = (int64_t)gridDim.x * (kEncThreads / 32);
  for (int64_t bt = (int64_t)blockIdx.x * (kEncThreads / 32) + wid; bt < nbatch; bt += wstep) {
    const int64_t first = bt * 32;
    const int cnt = p.items - first < 32 ? (int)(p.items - first) : 32;
    // ---- the batch's key rows into the stage (8-byte pieces; rows past the
    // end of the batch are not read)
    const uint2 *ksrc = reinterpret_cast<const uint2 *>(p.keys + first * kD);
    for (int e = lane; e < cnt * (kD / 4); e += 32) {
      const int r = e >> 5, c = e & 31;
      *reinterpret_cast<uint2 *>(stage + r * kEncRowStride + c * 8) = ksrc[e];
    }
    __syncwarp();
    // ---- this lane's item
    const int64_t item = first + lane;
    EncPlace pl{0, -1, 0, 0u, true};
    int bits = 0;
    uint64_t rec = 0;
    uint32_t st = 0u;
    if (lane < cnt) {
      pl = enc_place(p, item);
      if (!pl.skip) st = enc_record(p, pl, bits, rec);
    }
    const bool go = lane < cnt && !pl.skip && !st;
    if (st) set_err(p.err, st);
    const uint16_t *krow = reinterpret_cast<const uint16_t *>(stage + lane * kEncRowStride);
    if (go) {
      if (p.nu_ec)
        encode_key_lane_nu_bits(bits, krow, p.arena + rec, pl.slot, p.rad_lo[pl.h], p.rad_step[pl.h], sm.az_c2,
                                p.nu_ec, p.err);
      else
        encode_key_lane_bits(bits, krow, p.arena + rec, pl.slot, p.rad_lo[pl.h], p.rad_step[pl.h], sm.pol_c2,
                             sm.az_c2, p.err);
    }
    // ---- the value rows, the whole warp on each row; eight rows' loads are
    // issued before their stores, so their latencies overlap
    if (p.values) {
      const int64_t dst_row = go ? (((int64_t)pl.pid * p.Hkv + pl.h) * kPage + pl.slot) * kD : -1;
      constexpr int kRows = 8;
      for (int j0 = 0; j0 < cnt; j0 += kRows) {
        uint2 v[kRows];
        int64_t dr[kRows];
#pragma unroll
        for (int k = 0; k < kRows; ++k) {
          const int j = j0 + k;
          dr[k] = __shfl_sync(0xffffffffu, dst_row, j & 31);
          if (j >= cnt) dr[k] = -1;  // warp-uniform
          if (dr[k] >= 0) v[k] = *reinterpret_cast<const uint2 *>(p.values + (first + j) * kD + 4 * lane);
        }
#pragma unroll
        for (int k = 0; k < kRows; ++k)
          if (dr[k] >= 0) *reinterpret_cast<uint2 *>(p.v_pages + dr[k] + 4 * lane) = v[k];
      }
    }
    __syncwarp();
  }
}

// Few items (a decode step's appends): one warp per key, the warp form of
// the same arithmetic (encode_key_warp_seq), so no thread runs a whole key.
__global__ void __launch_bounds__(kEncThreads) encode_kernel_warp(const EncodeParams p) {
  __shared__ double pol_c2[kLutEntries], az_c2[kLutEntries];
  build_edge_tables(pol_c2, az_c2, threadIdx.x, kEncThreads, true);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (kEncThreads / 32) + (threadIdx.x >> 5);
  if (item >= p.items) return;
  const EncPlace pl = enc_place(p, item);
  if (pl.skip) return;
  int bits = 0;
  uint64_t rec = 0;
  const uint32_t st = enc_record(p, pl, bits, rec);
  if (st) {
    if (lane == 0) set_err(p.err, st);
    return;
  }
  encode_key_warp_seq_bits<true>(bits, p.keys + item * kD, p.arena + rec, pl.slot, p.rad_lo[pl.h], p.rad_step[pl.h],
                           pol_c2, az_c2, lane, p.err);
  if (p.values) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p.values + item * kD + 4 * lane);
    *reinterpret_cast<uint2 *>(p.v_pages + (((int64_t)pl.pid * p.Hkv + pl.h) * kPage + pl.slot) * kD + 4 * lane) = v;
  }
}

}  // namespace

// Checks shared by every entry point that reads an spkv_cache.
spkv_status check_cache(const spkv_cache *c) {
  if (!c) return SPKV_ERR_INVALID_ARG;
  if (c->head_dim != kD || c->page_size != kPage) return SPKV_ERR_UNSUPPORTED;
  if (c->num_kv_heads < 1 || c->num_pages < 0) return SPKV_ERR_INVALID_ARG;
  if (!c->code_arena || !c->hdr || !c->rad_lo_log2 || !c->rad_step_log2 || !c->v_pages)
    return SPKV_ERR_INVALID_ARG;
  if (((uintptr_t)c->code_arena & 15) || ((uintptr_t)c->v_pages & 15) || ((uintptr_t)c->hdr & 7))
    return SPKV_ERR_INVALID_ARG;
  return SPKV_OK;
}

int device_sm_count();

}  // namespace spkv

namespace spkv {
namespace {

spkv_status launch_encode(const spkv_cache *cache, EncodeParams &p, cudaStream_t stream) {
  p.arena = cache->code_arena;
  p.arena_bytes = cache->code_arena_bytes;
  p.hdr = cache->hdr;
  p.rad_lo = cache->rad_lo_log2;
  p.rad_step = cache->rad_step_log2;
  p.v_pages = cache->v_pages;
  p.err = cache->err_flags;
  p.Hkv = cache->num_kv_heads;
  p.num_pages = cache->num_pages;
  const int sms = device_sm_count();
  if (sms <= 0) return SPKV_ERR_CUDA;
  if (!p.nu_ec && p.items <= kEncWarpItems) {  // a decode step's appends: a warp per key
    const int grid = (int)((p.items + kEncThreads / 32 - 1) / (kEncThreads / 32));
    encode_kernel_warp<<<grid, kEncThreads, 0, stream>>>(p);
  } else {
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SPKV_ERR_CUDA;
    if (!configured[dev]) {
      if (cudaFuncSetAttribute(encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)sizeof(EncodeSmem)) != cudaSuccess)
        return SPKV_ERR_CUDA;
      configured[dev] = true;
    }
    // one wave of resident CTAs (3 per SM), each warp striding over batches of 32 items
    const int64_t batches = (p.items + 31) / 32;
    const int64_t want = (batches + kEncThreads / 32 - 1) / (kEncThreads / 32);
    const int grid = (int)(want < (int64_t)sms * 3 ? want : (int64_t)sms * 3);
    encode_kernel<<<grid, kEncThreads, sizeof(EncodeSmem), stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}

}  // namespace
}  // namespace spkv

extern "C" spkv_status spkv_encode_keys(const spkv_cache *cache, const uint16_t *keys, const uint16_t *values,
                                        const int32_t *start_pos, int32_t B, int32_t n_new,
                                        const int32_t *block_table, int32_t max_pages, void *stream) {
  using namespace spkv;
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  if (B < 0 || n_new < 0 || max_pages < 0) return SPKV_ERR_INVALID_ARG;
  if (B == 0 || n_new == 0) return SPKV_OK;
  if (!keys || !start_pos || !block_table || max_pages == 0) return SPKV_ERR_INVALID_ARG;
  if (((uintptr_t)keys & 7) || ((uintptr_t)values & 7)) return SPKV_ERR_INVALID_ARG;
  EncodeParams p = {};
  p.keys = keys;
  p.values = values;
  p.start_pos = start_pos;
  p.block_table = block_table;
  p.B = B;
  p.n_new = n_new;
  p.max_pages = max_pages;
  p.items = (int64_t)B * n_new * cache->num_kv_heads;
  return launch_encode(cache, p, (cudaStream_t)stream);
}

extern "C" spkv_status spkv_encode_keys_packed(const spkv_cache *cache, const uint16_t *keys, const uint16_t *values,
                                               const int32_t *seq_start, int32_t B, int64_t total_tokens,
                                               const int32_t *dst_pos, const int32_t *block_table, int32_t max_pages,
                                               void *stream) {
  using namespace spkv;
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  if (B < 0 || total_tokens < 0 || max_pages < 0) return SPKV_ERR_INVALID_ARG;
  if (B == 0 || total_tokens == 0) return SPKV_OK;
  if (!keys || !seq_start || !dst_pos || !block_table || max_pages == 0) return SPKV_ERR_INVALID_ARG;
  if (((uintptr_t)keys & 7) || ((uintptr_t)values & 7)) return SPKV_ERR_INVALID_ARG;
  EncodeParams p = {};
  p.keys = keys;
  p.values = values;
  p.seq_start = seq_start;
  p.dst_pos = dst_pos;
  p.block_table = block_table;
  p.B = B;
  p.n_new = 0;
  p.max_pages = max_pages;
  p.items = total_tokens * cache->num_kv_heads;
  return launch_encode(cache, p, (cudaStream_t)stream);
}

extern "C" spkv_status spkv_encode_keys_nonuniform(const spkv_cache *cache, const uint16_t *keys,
                                                   const uint16_t *values, const int32_t *start_pos, int32_t B,
                                                   int32_t n_new, const int32_t *block_table, int32_t max_pages,
                                                   int32_t bits, const double *edge_cos, void *stream) {
  using namespace spkv;
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  if (B < 0 || n_new < 0 || max_pages < 0) return SPKV_ERR_INVALID_ARG;
  if (tier_of_bits(bits) < 0) return SPKV_ERR_UNSUPPORTED;
  if (!edge_cos || ((uintptr_t)edge_cos & 7)) return SPKV_ERR_INVALID_ARG;
  if (B == 0 || n_new == 0) return SPKV_OK;
  if (!keys || !start_pos || !block_table || max_pages == 0) return SPKV_ERR_INVALID_ARG;
  if (((uintptr_t)keys & 7) || ((uintptr_t)values & 7)) return SPKV_ERR_INVALID_ARG;
  EncodeParams p = {};
  p.keys = keys;
  p.values = values;
  p.start_pos = start_pos;
  p.block_table = block_table;
  p.B = B;
  p.n_new = n_new;
  p.max_pages = max_pages;
  p.items = (int64_t)B * n_new * cache->num_kv_heads;
  p.nu_ec = edge_cos;
  p.nu_bits = bits;
  return launch_encode(cache, p, (cudaStream_t)stream);
}
