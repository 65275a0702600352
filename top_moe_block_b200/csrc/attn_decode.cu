// Decode attention: one new query token per sequence over the sliding
// window of the KV cache (keys max(0, t - window + 1) .. t), GQA with the
// rep = n_q / n_kv query heads of a kv head processed together so every K/V
// byte is read once (nnterp "zaya" page: grouped-query eager attention).
//
// HBM-bound (the window's K and V: 2 x d x 2 bytes per key and kv head).
// Split-KV: CTA (chunk, kv head, sequence) covers 256 keys, 4 warps of 64.
// Each lane owns d/32 dims: it streams 8-byte slices of the keys (a warp
// reads whole 256-byte rows, coalesced), forms rep partial dot products per
// key, and a butterfly reduce-scatter over the warp leaves one complete
// (key, head) score per lane.  Online softmax per head, P.V accumulated on
// the lane's own dims.  A second kernel merges the chunks.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

constexpr int kChunk = 256;   // keys per CTA up to kMaxChunks chunks (longer spans: longer chunks)
constexpr int kWarps = 4;
constexpr int kMaxChunks = 64; // a head's partials in the workspace

template <int D, int REP>
__global__ void __launch_bounds__(128) attn_decode_kernel(const DecodeAttnParams p) {
  constexpr int DPL = D / 32;
  constexpr int KPG = 32 / REP;  // keys per group: KPG * REP == 32 scores per warp step
  griddep_begin();
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  // A position outside the cache (already reported by the conv kernel) gives
  // an empty key range, so nothing outside the cache is read.
  const int t_raw = p.cache_len[b];
  const int t = (t_raw >= 0 && t_raw < p.cap) ? t_raw : -1;
  const int lo = max(0, t - p.window + 1);
  const int c_begin = lo + chunk * p.chunk_keys;
  const int c_end = min(t + 1, c_begin + p.chunk_keys);
  const int w_begin = c_begin + warp * (p.chunk_keys / kWarps);
  const int w_end = min(c_end, w_begin + p.chunk_keys / kWarps);

  const float sl2 = p.scale * 1.4426950408889634f;
  float q[REP][DPL];
  const auto* qg = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.n_q + g * REP) * D + lane * DPL;
#pragma unroll
  for (int hh = 0; hh < REP; ++hh)
#pragma unroll
    for (int i = 0; i < DPL; ++i) q[hh][i] = bf2f(qg[hh * D + i]) * sl2;

  const auto* Kg = static_cast<const __nv_bfloat16*>(p.k_cache) + ((size_t)b * p.n_kv + g) * p.cap * D + lane * DPL;
  const auto* Vg = static_cast<const __nv_bfloat16*>(p.v_cache) + ((size_t)b * p.n_kv + g) * p.cap * D + lane * DPL;

  float o[REP][DPL];
#pragma unroll
  for (int hh = 0; hh < REP; ++hh)
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[hh][i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;  // for head (lane % REP)

  for (int base = w_begin; base < w_end; base += KPG) {
    float kf[KPG][DPL], vf[KPG][DPL];
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk) {
      const int key = base + kk;
      if (key < w_end) {
        if constexpr (DPL == 4) {
          const uint2 ku = *reinterpret_cast<const uint2*>(Kg + (size_t)key * D);
          const uint2 vu = *reinterpret_cast<const uint2*>(Vg + (size_t)key * D);
          const float2 k01 = unpack_bf2(ku.x), k23 = unpack_bf2(ku.y);
          const float2 v01 = unpack_bf2(vu.x), v23 = unpack_bf2(vu.y);
          kf[kk][0] = k01.x; kf[kk][1] = k01.y; kf[kk][2] = k23.x; kf[kk][3] = k23.y;
          vf[kk][0] = v01.x; vf[kk][1] = v01.y; vf[kk][2] = v23.x; vf[kk][3] = v23.y;
        } else {
          const uint32_t ku = *reinterpret_cast<const uint32_t*>(Kg + (size_t)key * D);
          const uint32_t vu = *reinterpret_cast<const uint32_t*>(Vg + (size_t)key * D);
          const float2 k01 = unpack_bf2(ku), v01 = unpack_bf2(vu);
          kf[kk][0] = k01.x; kf[kk][1] = k01.y;
          vf[kk][0] = v01.x; vf[kk][1] = v01.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) kf[kk][i] = vf[kk][i] = 0.f;
      }
    }
    // partial scores, value index = kk * REP + hh
    float v[32];
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk)
#pragma unroll
      for (int hh = 0; hh < REP; ++hh) {
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) a = fmaf(q[hh][i], kf[kk][i], a);
        v[kk * REP + hh] = a;
      }
    // butterfly reduce-scatter: lane l ends with the full sum of value l
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
      const bool upper = (lane & s) != 0;
#pragma unroll
      for (int i = 0; i < s; ++i) {
        const float send = upper ? v[i] : v[i + s];
        const float keep = upper ? v[i + s] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
      }
    }
    const int my_key = base + lane / REP;
    float sc = (my_key < w_end) ? v[0] : -INFINITY;
    float gm = sc;
#pragma unroll
    for (int s = REP; s < 32; s <<= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, s));
    const float m_new = fmaxf(m_run, gm);
    const float bse = (m_new == -INFINITY) ? 0.f : m_new;
    const float pk = exp2f(sc - bse);
    float ps = pk;
#pragma unroll
    for (int s = REP; s < 32; s <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, s);
    const float corr = exp2f(m_run - bse);
    l_run = l_run * corr + ps;
    m_run = m_new;
#pragma unroll
    for (int hh = 0; hh < REP; ++hh) {
      const float ch = __shfl_sync(0xffffffffu, corr, hh);
#pragma unroll
      for (int i = 0; i < DPL; ++i) o[hh][i] *= ch;
    }
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk)
#pragma unroll
      for (int hh = 0; hh < REP; ++hh) {
        const float pv = __shfl_sync(0xffffffffu, pk, kk * REP + hh);
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[hh][i] = fmaf(pv, vf[kk][i], o[hh][i]);
      }
  }

  // merge the 4 warps of this CTA, then write the chunk's partial result
  __shared__ float sm_m[kWarps][REP], sm_l[kWarps][REP];
  __shared__ float sm_o[kWarps][REP][D];
  if (lane < REP) {
    sm_m[warp][lane] = m_run;
    sm_l[warp][lane] = l_run;
  }
#pragma unroll
  for (int hh = 0; hh < REP; ++hh)
#pragma unroll
    for (int i = 0; i < DPL; ++i) sm_o[warp][hh][lane * DPL + i] = o[hh][i];
  __syncthreads();
  const size_t part_idx = (((size_t)b * p.n_kv + g) * p.n_chunks + chunk) * REP;
  float* pm = p.part;                                           // [.., REP] max
  float* pl = p.part + (size_t)p.B * p.n_kv * p.n_chunks * REP; // [.., REP] sum
  float* po = pl + (size_t)p.B * p.n_kv * p.n_chunks * REP;     // [.., REP, D]
  for (int idx = threadIdx.x; idx < REP * D; idx += blockDim.x) {
    const int hh = idx / D, dd = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][hh]);
    const float bse = (M == -INFINITY) ? 0.f : M;
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = exp2f(sm_m[w][hh] - bse);
      L += sm_l[w][hh] * f;
      O += sm_o[w][hh][dd] * f;
    }
    po[(part_idx + hh) * D + dd] = O;
    if (dd == 0) {
      pm[part_idx + hh] = M;
      pl[part_idx + hh] = L;
    }
  }
}

template <int D>
__global__ void attn_decode_combine(const DecodeAttnParams p, int rep) {
  griddep_begin();
  const int bh = blockIdx.x;
  const int b = bh / p.n_q, h = bh % p.n_q;
  const int g = h / rep, hh = h % rep;
  const int dd = threadIdx.x;
  const float* pm = p.part;
  const float* pl = p.part + (size_t)p.B * p.n_kv * p.n_chunks * rep;
  const float* po = pl + (size_t)p.B * p.n_kv * p.n_chunks * rep;
  float M = -INFINITY;
  for (int c = 0; c < p.n_chunks; ++c) M = fmaxf(M, pm[(((size_t)b * p.n_kv + g) * p.n_chunks + c) * rep + hh]);
  const float bse = (M == -INFINITY) ? 0.f : M;
  float L = 0.f, O = 0.f;
  for (int c = 0; c < p.n_chunks; ++c) {
    const size_t i = (((size_t)b * p.n_kv + g) * p.n_chunks + c) * rep + hh;
    const float f = exp2f(pm[i] - bse);
    L += pl[i] * f;
    O += po[i * D + dd] * f;
  }
  auto* out = static_cast<__nv_bfloat16*>(p.out);
  out[(size_t)b * p.n_q * D + h * D + dd] = f2bf(L > 0.f ? O / L : 0.f);
}

}  // namespace

int decode_attn_max_chunks(int window) {
  const long n = ((long)window + kChunk - 1) / kChunk;
  return n < 1 ? 1 : (n > kMaxChunks ? kMaxChunks : (int)n);
}

size_t decode_attn_ws_bytes(int B, int n_q, int d, int max_chunks) {
  return (size_t)B * n_q * max_chunks * (d + 2) * sizeof(float);
}

void decode_attn_split(int span, int max_chunks, int* n_chunks, int* chunk_keys) {
  int n = (span + kChunk - 1) / kChunk;
  int ck = kChunk;
  if (n > max_chunks) {   // longer chunks, still whole multiples of 256 keys
    ck = ((span + max_chunks - 1) / max_chunks + kChunk - 1) / kChunk * kChunk;
    n = (span + ck - 1) / ck;
  }
  *n_chunks = n < 1 ? 1 : n;
  *chunk_keys = ck;
}

int launch_attn_decode(const DecodeAttnParams& p, cudaStream_t st) {
  if (p.B <= 0) return ZAYA_OK;
  if (p.n_chunks < 1 || p.n_chunks > kMaxChunks || p.chunk_keys % kChunk) return ZAYA_ERR_UNSUPPORTED;
  const int rep = p.n_q / p.n_kv;
  const dim3 grid(p.n_chunks, p.n_kv, p.B);
#define ZAYA_DEC(DV, RV)                                                   \
  if (p.d == DV && rep == RV) {                                            \
    launch_k(attn_decode_kernel<DV, RV>, grid, dim3(32 * kWarps), 0, st, nullptr, 0, p);          \
    launch_k(attn_decode_combine<DV>, dim3(p.B * p.n_q), dim3(DV), 0, st, nullptr, 0, p, RV);   \
    return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;    \
  }
  ZAYA_DEC(128, 4)
  ZAYA_DEC(64, 4)
  ZAYA_DEC(128, 2)
  ZAYA_DEC(64, 2)
  ZAYA_DEC(128, 1)
  ZAYA_DEC(64, 1)
  ZAYA_DEC(128, 8)
  ZAYA_DEC(64, 8)
#undef ZAYA_DEC
  return ZAYA_ERR_UNSUPPORTED;
}

}  // namespace zaya
