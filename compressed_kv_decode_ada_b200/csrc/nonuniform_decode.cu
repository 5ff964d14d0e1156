// nonuniform_decode.cu -- ADA decode attention over a cache encoded with the
// non-uniform angle quantiser (spkv_encode_keys_nonuniform).
//
// Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
// for Efficient Long-Context Inference", technical summary section 2.1: f_b
// is the cosine of the decoded angles, u~_j = (prod_{m<j} sin phi_m) cos phi_j
// (u~_127 = the product of all 127 sines), logits ||q|| r~ f_b / sqrt(d),
// softmax over the retained tokens, then P.V.  The pages leave the quantiser
// open; this variant's cells are the equal-probability cells of each polar
// angle's sin^(d-1-i) law (spkv_nonuniform_tables), reconstructed at the cell
// medians; the azimuth keeps the uniform cells.  The query is coded with the
// same quantiser at the cache's b (as the uniform path codes it).
//
// Structure: a prep kernel turns the fp64 median tables into one fp32
// (cos, sin) table of 127 x 2^b entries (the azimuth's uniform medians in its
// last row); one CTA per (sequence, kv head, split) codes the G query heads,
// runs f_b for 32 tokens per warp at a time (lane = token, the slot's code
// words in registers), an online softmax and P.V on CUDA cores, and writes
// the split's partial record per query head; spkv_merge_partials combines
// the splits.
#include <cfloat>

#include "spkv_encode.cuh"

namespace spkv {
spkv_status check_cache(const spkv_cache *c);
int device_sm_count();

namespace {

constexpr int kNuThreads = 128;  // 4 warps
constexpr int kNuWarps = kNuThreads / 32;
constexpr int kNuMaxG = 8;
constexpr int kRec = 132;  // floats per partial record (M, L, 0, 0, o[128])

// ---- (cos, sin) table: rows 0..125 the polar medians, row 126 the azimuth's
// uniform medians (c + 1/2) 2 pi / 2^b
__global__ void nu_table_kernel(const double *mid_cos, const double *mid_sin, int n, float2 *tab) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 127 * n) return;
  const int row = i / n, c = i - row * n;
  if (row < 126) {
    tab[i] = make_float2((float)mid_cos[i], (float)mid_sin[i]);
  } else {
    double s, co;
    sincospi((2.0 * c + 1.0) / (double)n, &s, &co);  // angle (c + 1/2) 2 pi / n
    tab[i] = make_float2((float)co, (float)s);
  }
}

// The query's 127 codes with the non-uniform quantiser (one thread): the
// suffix sums in encode_key_lane's order, polar codes against each angle's
// edges, the uniform azimuth; returns ||q||^2.
template <int BITS>
__device__ double nu_query_codes(const uint16_t *q, const double *ec, const double *ac2, uint8_t *codes) {
  constexpr int NE = (1 << BITS) - 1;
  const uint2 *kr = reinterpret_cast<const uint2 *>(q);
  double x[4], s[4], T = 0.0;
  for (int g = 31; g >= 0; --g) {
    bf16x4_to_f64(kr[g], x);
    s[3] = x[3] * x[3];
    s[2] = fma(x[2], x[2], s[3]);
    s[1] = fma(x[1], x[1], s[2]);
    s[0] = fma(x[0], x[0], s[1]);
    const double Tn = T;
    T = s[0] + Tn;
#pragma unroll
    for (int k = 3; k >= 0; --k) {
      const int a = 4 * g + k;
      int c = 0;
      if (a < 126) c = polar_code_nu<BITS>(x[k], s[k] + Tn, ec + a * NE);
      else if (a == 126) c = azimuth_code<BITS>(x[2], x[3], s[2] + Tn, ac2);
      if (a < 127) codes[a] = (uint8_t)c;
    }
  }
  return T;
}

struct NuParams {
  const uint8_t *arena;
  uint64_t arena_bytes;
  const spkv_page_hdr *hdr;
  const float *rad_lo, *rad_step;
  const uint16_t *v_pages;
  const uint16_t *keep;
  uint32_t *err;
  int Hkv, num_pages;
  const double *ec;   // polar edge cosines [126][2^b - 1] (query coding)
  const float2 *tab;  // (cos, sin) [127][2^b]
  const uint16_t *q;
  int B, Hq;
  const int32_t *block_table;
  int max_pages;
  const int32_t *ctx_lens;
  int max_ctx;
  int S;          // splits per (sequence, kv head) row
  float *records;  // [S, B, Hq, 132]
  float *logits;   // optional [B, Hq, max_ctx], natural-log units
};

// Code of angle j from the slot's words (chunk c's 4 words in wv[c]).
template <int BITS>
__device__ __forceinline__ uint32_t nu_word(const uint4 (&wv)[BITS], int w) {
  const uint4 v = wv[w >> 2];
  const int k = w & 3;
  return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
}
template <int BITS>
__device__ __forceinline__ uint32_t nu_code(const uint4 (&wv)[BITS], int j) {
  const int o = j * BITS, w = o >> 5, sh = o & 31;
  uint32_t v = nu_word<BITS>(wv, w) >> sh;
  if (sh + BITS > 32) v |= nu_word<BITS>(wv, w + 1) << (32 - sh);
  return v & ((1u << BITS) - 1u);
}

template <int BITS, int G>
__global__ void __launch_bounds__(kNuThreads) nu_decode_kernel(const NuParams p) {
  constexpr int N = 1 << BITS;
  __shared__ double pol_c2[kLutEntries], az_c2[kLutEntries];
  __shared__ __align__(16) float uq[128][G];
  __shared__ float qs[G];
  __shared__ uint8_t qcodes[G][128];
  __shared__ float wm[kNuWarps][G], wl[kNuWarps][G];
  __shared__ float wacc[kNuWarps][G][128];
  // b <= 4: the (cos, sin) table in shared memory (one angle's 2^b entries
  // are one 64- or 128-byte row, so a warp's lookups of one angle never
  // conflict); wider tables are read through L1
  constexpr bool kSmemTab = BITS <= 4;
  __shared__ float2 stab[kSmemTab ? 127 * N : 1];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int row = blockIdx.x / p.S, split = blockIdx.x - row * p.S;
  const int b = row / p.Hkv, h = row - b * p.Hkv;
  int ctx = p.ctx_lens[b];
  if (ctx < 0 || ctx > p.max_ctx || ctx > p.max_pages * kPage) {
    if (split == 0 && h == 0 && tid == 0) set_err(p.err, SPKV_DEVERR_CTX);
    ctx = 0;
  }
  const int np = (ctx + kPage - 1) / kPage;
  const int pg0 = (int)((int64_t)split * np / p.S), pg1 = (int)((int64_t)(split + 1) * np / p.S);
  const int t_begin = pg0 * kPage, t_end = min(pg1 * kPage, ctx);

  build_edge_tables(pol_c2, az_c2, tid, kNuThreads);
  if constexpr (kSmemTab)
    for (int i = tid; i < 127 * N; i += kNuThreads) stab[i] = __ldg(p.tab + i);
  __syncthreads();
  if (tid < G) {  // the query heads' codes and scales (log2 units)
    const double n2 = nu_query_codes<BITS>(p.q + ((int64_t)b * p.Hq + h * G + tid) * kD, p.ec,
                                            az_c2 + lut_off(tier_of_bits(BITS)), qcodes[tid]);
    qs[tid] = n2 > 0.0 ? (float)(sqrt(n2) * 1.4426950408889634 / sqrt(128.0)) : 0.0f;
  }
  __syncthreads();
  if (tid < G) {  // u~ of the coded query
    float P = 1.0f;
    for (int j = 0; j < 127; ++j) {
      const float2 cs = p.tab[j * N + qcodes[tid][j]];
      uq[j][tid] = P * cs.x;
      P *= cs.y;
    }
    uq[127][tid] = P;
  }
  __syncthreads();

  float m[G], l[G], acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.0f;
    acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.0f;
  }
  const float Lh = p.rad_lo[h], Dh = p.rad_step[h];
  for (int t0 = t_begin + wid * 32; t0 < t_end; t0 += kNuThreads) {
    const int t = t0 + lane;
    const int slot = t & (kPage - 1);
    int pid = -1;
    bool ok = false;
    uint64_t rec = 0;
    if (t < t_end) {
      pid = p.block_table[(int64_t)b * p.max_pages + (t >> 4)];
      if (pid < 0 || pid >= p.num_pages) {
        set_err(p.err, SPKV_DEVERR_PAGE_ID);
      } else {
        const spkv_page_hdr hd = p.hdr[pid];
        if (hd.bits != BITS) {
          set_err(p.err, SPKV_DEVERR_BITS);
        } else {
          rec = (uint64_t)hd.code_off16 * 16u + (uint64_t)h * rec_bytes(BITS);
          if (rec + rec_bytes(BITS) > p.arena_bytes) set_err(p.err, SPKV_DEVERR_RECORD);
          else ok = !p.keep || ((p.keep[(int64_t)pid * p.Hkv + h] >> slot) & 1u);
        }
      }
    }
    float x[G];
#pragma unroll
    for (int g = 0; g < G; ++g) x[g] = -INFINITY;
    if (ok) {
      uint4 wv[BITS];
#pragma unroll
      for (int c = 0; c < BITS; ++c) wv[c] = *reinterpret_cast<const uint4 *>(p.arena + rec + (c * 16 + slot) * 16);
      const float r = exp2f(fmaf((float)p.arena[rec + 256 * BITS + slot], Dh, Lh));
      // two independent chains, angles 0 .. 63 (A) and 64 .. 126 (B, its
      // products of sines started at 1), joined as f = A + P_A (B + u_q,127 P_B)
      float fa[G], fb[G];
#pragma unroll
      for (int g = 0; g < G; ++g) fa[g] = fb[g] = 0.0f;
      float Pa = 1.0f, Pb = 1.0f;
      auto entry = [&](int j) -> float2 {
        const int e = j * N + (int)nu_code<BITS>(wv, j);
        if constexpr (kSmemTab) return stab[e];
        else return __ldg(p.tab + e);
      };
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const float2 ca = entry(j);
        const float ua = Pa * ca.x;
        Pa *= ca.y;
#pragma unroll
        for (int g = 0; g < G; ++g) fa[g] = fmaf(uq[j][g], ua, fa[g]);
        if (j < 63) {
          const float2 cb = entry(64 + j);
          const float ub = Pb * cb.x;
          Pb *= cb.y;
#pragma unroll
          for (int g = 0; g < G; ++g) fb[g] = fmaf(uq[64 + j][g], ub, fb[g]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) x[g] = qs[g] * r * fmaf(Pa, fmaf(uq[127][g], Pb, fb[g]), fa[g]);
    }
    if (p.logits && t < t_end) {
#pragma unroll
      for (int g = 0; g < G; ++g)
        p.logits[((int64_t)b * p.Hq + h * G + g) * p.max_ctx + t] = ok ? x[g] * 0.6931471805599453f : -INFINITY;
    }
    // ---- online softmax over the chunk (log2 units), then P.V
    float pv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = x[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mn = fmaxf(m[g], mx);
      const float alpha = (m[g] == -INFINITY || mn == -INFINITY) ? (m[g] == -INFINITY ? 0.0f : 1.0f)
                                                                  : exp2f(m[g] - mn);
      pv[g] = x[g] == -INFINITY ? 0.0f : exp2f(x[g] - mn);
      float ps = pv[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l[g] = l[g] * alpha + ps;
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[g][k] *= alpha;
      m[g] = mn;
    }
    // P.V: lane l holds dims 4 l .. 4 l + 3; the chunk's value rows are
    // loaded eight at a time before their products, so the loads overlap
    const unsigned okm = __ballot_sync(0xffffffffu, ok);
    // this lane's token's value row (element offset), or -1
    const int64_t vrow = ok ? (((int64_t)pid * p.Hkv + h) * kPage + slot) * kD : -1;
    for (int i0 = 0; i0 < 32; i0 += 8) {
      if (!((okm >> i0) & 0xffu)) continue;  // warp-uniform
      uint2 vr[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int64_t o = __shfl_sync(0xffffffffu, vrow, i0 + k);
        vr[k] = o >= 0 ? *reinterpret_cast<const uint2 *>(p.v_pages + o + 4 * lane) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float v0 = bf16lo(vr[k].x), v1 = bf16hi(vr[k].x), v2 = bf16lo(vr[k].y), v3 = bf16hi(vr[k].y);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pg = __shfl_sync(0xffffffffu, pv[g], i0 + k);  // 0 for a token not decoded
          acc[g][0] = fmaf(pg, v0, acc[g][0]);
          acc[g][1] = fmaf(pg, v1, acc[g][1]);
          acc[g][2] = fmaf(pg, v2, acc[g][2]);
          acc[g][3] = fmaf(pg, v3, acc[g][3]);
        }
      }
    }
  }
  // ---- the split's record per query head: the warps combined
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (lane == 0) {
      wm[wid][g] = m[g];
      wl[wid][g] = l[g];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) wacc[wid][g][4 * lane + k] = acc[g][k];
  }
  __syncthreads();
  for (int idx = tid; idx < G * kD; idx += kNuThreads) {
    const int g = idx / kD, d = idx - g * kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kNuWarps; ++w) M = fmaxf(M, wm[w][g]);
    float L = 0.0f, o = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kNuWarps; ++w) {
        if (wm[w][g] == -INFINITY) continue;
        const float s = exp2f(wm[w][g] - M);
        L = fmaf(s, wl[w][g], L);
        o = fmaf(s, wacc[w][g][d], o);
      }
      o = L > 0.0f ? o / L : 0.0f;
    }
    float *rp = p.records + (((int64_t)split * p.B + b) * p.Hq + h * G + g) * kRec;
    rp[4 + d] = o;
    if (d == 0) {
      rp[0] = M;
      rp[1] = L;
      rp[2] = 0.0f;
      rp[3] = 0.0f;
    }
  }
}

// Splits per (sequence, kv head) row: explicit, or about kNuCtasPerSM CTAs
// per SM in all (the CTA is small: several per SM keep its latency-bound
// token loop fed), at most one per page.  0 on a device error.
constexpr int kNuCtasPerSM = 6;
int nu_splits(int B, int Hkv, int max_ctx, int num_splits) {
  if (num_splits > 0) return num_splits;
  const int sms = device_sm_count();
  if (sms <= 0) return 0;
  const int64_t rows = (int64_t)B * Hkv;
  int64_t S = rows > 0 ? (kNuCtasPerSM * (int64_t)sms + rows - 1) / rows : 1;
  const int64_t pages = ((int64_t)max_ctx + kPage - 1) / kPage;
  if (S > pages) S = pages;
  return (int)(S < 1 ? 1 : S);
}

size_t nu_records_bytes(int B, int Hq, int S) { return ((size_t)S * B * Hq * kRec * 4 + 255) / 256 * 256; }

template <int BITS, int G>
void launch_nu(const NuParams &p, cudaStream_t stream) {
  nu_decode_kernel<BITS, G><<<p.B * p.Hkv * p.S, kNuThreads, 0, stream>>>(p);
}

template <int BITS>
bool launch_nu_g(int G, const NuParams &p, cudaStream_t stream) {
  switch (G) {
    case 1: launch_nu<BITS, 1>(p, stream); return true;
    case 2: launch_nu<BITS, 2>(p, stream); return true;
    case 4: launch_nu<BITS, 4>(p, stream); return true;
    case 8: launch_nu<BITS, 8>(p, stream); return true;
  }
  return false;
}

}  // namespace
}  // namespace spkv

using namespace spkv;

extern "C" size_t spkv_decode_nonuniform_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t max_ctx,
                                                         int32_t num_splits, int32_t bits) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || max_ctx < 0 || num_splits < 0 || tier_of_bits(bits) < 0) return 0;
  const int S = nu_splits(B, Hkv, max_ctx, num_splits);
  if (S < 1) return 0;
  return nu_records_bytes(B, Hq, S) + (size_t)127 * (1u << bits) * sizeof(float2);
}

extern "C" spkv_status spkv_decode_attention_nonuniform(const spkv_cache *cache, const uint16_t *q, int32_t B,
                                                        int32_t Hq, const int32_t *block_table, int32_t max_pages,
                                                        const int32_t *ctx_lens, int32_t max_ctx, int32_t bits,
                                                        const double *edge_cos, const double *mid_cos,
                                                        const double *mid_sin, void *out, int32_t out_is_bf16,
                                                        float *logits, void *ws, size_t ws_bytes,
                                                        int32_t num_splits, void *stream) {
  spkv_status st = check_cache(cache);
  if (st != SPKV_OK) return st;
  const int Hkv = cache->num_kv_heads;
  if (B < 0 || Hq < 1 || max_pages < 0 || max_ctx < 0 || num_splits < 0) return SPKV_ERR_INVALID_ARG;
  if (Hq % Hkv) return SPKV_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SPKV_ERR_UNSUPPORTED;
  if (tier_of_bits(bits) < 0) return SPKV_ERR_UNSUPPORTED;
  if (!edge_cos || !mid_cos || !mid_sin || ((uintptr_t)edge_cos & 7) || ((uintptr_t)mid_cos & 7) ||
      ((uintptr_t)mid_sin & 7))
    return SPKV_ERR_INVALID_ARG;
  if (B == 0) return SPKV_OK;
  if (!q || !block_table || !ctx_lens || !out || ((uintptr_t)q & 7) || ((uintptr_t)out & 15) || (logits && ((uintptr_t)logits & 3)))
    return SPKV_ERR_INVALID_ARG;
  const int S = nu_splits(B, Hkv, max_ctx, num_splits);
  if (S < 1) return SPKV_ERR_CUDA;
  if ((int64_t)B * Hkv * S > 0x7fffffff) return SPKV_ERR_UNSUPPORTED;
  const size_t rec_bytes_all = nu_records_bytes(B, Hq, S);
  const size_t need = rec_bytes_all + (size_t)127 * (1u << bits) * sizeof(float2);
  if (!ws || ((uintptr_t)ws & 255) || ws_bytes < need) return SPKV_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  NuParams p;
  p.arena = cache->code_arena;
  p.arena_bytes = cache->code_arena_bytes;
  p.hdr = cache->hdr;
  p.rad_lo = cache->rad_lo_log2;
  p.rad_step = cache->rad_step_log2;
  p.v_pages = cache->v_pages;
  p.keep = cache->keep_mask;
  p.err = cache->err_flags;
  p.Hkv = Hkv;
  p.num_pages = cache->num_pages;
  p.ec = edge_cos;
  p.records = reinterpret_cast<float *>(ws);
  p.tab = reinterpret_cast<const float2 *>(reinterpret_cast<uint8_t *>(ws) + rec_bytes_all);
  p.q = q;
  p.B = B;
  p.Hq = Hq;
  p.block_table = block_table;
  p.max_pages = max_pages;
  p.ctx_lens = ctx_lens;
  p.max_ctx = max_ctx;
  p.S = S;
  p.logits = logits;
  const int n = 1 << bits;
  nu_table_kernel<<<(127 * n + 255) / 256, 256, 0, s>>>(mid_cos, mid_sin, n,
                                                        const_cast<float2 *>(p.tab));
  switch (bits) {
    case 3: launch_nu_g<3>(G, p, s); break;
    case 4: launch_nu_g<4>(G, p, s); break;
    case 6: launch_nu_g<6>(G, p, s); break;
    default: launch_nu_g<8>(G, p, s); break;
  }
  if (cudaGetLastError() != cudaSuccess) return SPKV_ERR_CUDA;
  return spkv_merge_partials(p.records, S, B, Hq, out, out_is_bf16, stream);
}
