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
// reaches (binary search over the 2^b - 1 edges), i.e. floor(phi 2^b / pi)
// clamped to 2^b - 1 -- ties go to the upper cell.  The azimuth (angle 127,
// range [0, 2 pi)) uses the same test on (x_126, x_127) with the half-plane
// given by the sign of x_127.  The radius code uses fp64 log2.
#include "spkv_encode.cuh"

namespace spkv {
namespace {

constexpr int kEncThreads = 256;
constexpr int kEncWarps = kEncThreads / 32;

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
};

struct EncodeSmem {
  double pol_c2[kLutEntries];
  double az_c2[kLutEntries];
  uint8_t codes[kEncWarps][128];
};

__global__ void __launch_bounds__(kEncThreads) encode_kernel(const EncodeParams p) {
  __shared__ EncodeSmem sm;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  build_edge_tables(sm.pol_c2, sm.az_c2, tid, kEncThreads);
  __syncthreads();

  const int64_t nwarps = (int64_t)gridDim.x * kEncWarps;
  for (int64_t item = (int64_t)blockIdx.x * kEncWarps + wid; item < p.items; item += nwarps) {
    const int h = (int)(item % p.Hkv);
    const int64_t bn = item / p.Hkv;
    int b, pos;
    if (p.dst_pos) {  // token bn of the concatenated sequences, to dst_pos[bn]
      pos = p.dst_pos[bn];
      if (pos < 0) continue;
      int lo = 0, hi = p.B;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)p.seq_start[mid] <= bn) lo = mid;
        else hi = mid;
      }
      b = lo;
      if (bn < (int64_t)p.seq_start[b] || bn >= (int64_t)p.seq_start[b + 1]) {
        if (lane == 0) set_err(p.err, SPKV_DEVERR_CTX);
        continue;
      }
    } else {
      b = (int)(bn / p.n_new);
      pos = p.start_pos[b] + (int)(bn % p.n_new);
    }
    if (pos < 0 || pos >= p.max_pages * kPage) {
      if (lane == 0) set_err(p.err, SPKV_DEVERR_CTX);
      continue;
    }
    const int pid = p.block_table[(int64_t)b * p.max_pages + pos / kPage];
    if (pid < 0 || pid >= p.num_pages) {
      if (lane == 0) set_err(p.err, SPKV_DEVERR_PAGE_ID);
      continue;
    }
    const spkv_page_hdr hd = p.hdr[pid];
    const int bits = hd.bits;
    if (tier_of_bits(bits) < 0) {
      if (lane == 0) set_err(p.err, SPKV_DEVERR_BITS);
      continue;
    }
    const uint64_t rec = (uint64_t)hd.code_off16 * 16u + (uint64_t)h * rec_bytes(bits);
    if (rec + rec_bytes(bits) > p.arena_bytes) {
      if (lane == 0) set_err(p.err, SPKV_DEVERR_RECORD);
      continue;
    }
    const int slot = pos % kPage;

    encode_key_warp(p.keys + item * kD, bits, p.arena + rec, slot, p.rad_lo[h], p.rad_step[h], sm.pol_c2, sm.az_c2,
                    sm.codes[wid], lane, p.err);
    // ---- value row (optional)
    if (p.values) {
      const uint2 v = *reinterpret_cast<const uint2 *>(p.values + item * kD + 4 * lane);
      uint16_t *dst = p.v_pages + (((int64_t)pid * p.Hkv + h) * kPage + slot) * kD + 4 * lane;
      *reinterpret_cast<uint2 *>(dst) = v;
    }
    __syncwarp();
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
  const int64_t want = (p.items + kEncWarps - 1) / kEncWarps;
  const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  encode_kernel<<<grid, kEncThreads, 0, stream>>>(p);
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
