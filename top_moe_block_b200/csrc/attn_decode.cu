// Decode attention: one new query token per sequence over the sliding
// window of the KV cache (keys max(0, t - window + 1) .. t), GQA with the
// rep = n_q / n_kv query heads of a kv head processed together so every K/V
// byte is read once (nnterp "zaya" page: grouped-query eager attention).
//
// HBM-bound (the window's K and V: 2 x d x 2 bytes per key and kv head).
// Split-KV: CTA (chunk, kv head, sequence) covers chunk_keys keys, 4 warps of
// a quarter each.  A warp streams its keys in 16-key slices (K and V rows by
// cp.async into a two-slot ring, 16-byte chunks XOR-swizzled by key so the
// ldmatrix reads are free of bank conflicts) and runs both products on the
// tensor cores with mma.sync m16n8k16 (bf16 in, fp32 accumulate): the rep
// query heads are the rows of A (padded to 16), S = Q K^T in fp32, online
// softmax per row on the accumulator fragments, P rounded to bf16 becomes the
// A operand of P V straight from registers, V read with ldmatrix.trans.  The
// four warps' (max, sum, O) are merged in shared memory into the chunk's
// partial; a second kernel merges the chunks.
// An fp8 cache (E4M3 bytes): the slice's raw bytes stream into a two-slot
// staging ring (half the bytes), each warp converts its slice to f16 (exact)
// in the swizzled layout above, and both products run on f16 mma.sync with q
// and P as f16 (q's bf16 values are exact in f16 within its range, P gains
// precision).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

constexpr int kChunk = 256;   // keys per CTA up to kMaxChunks chunks (longer spans: longer chunks)
constexpr int kWarps = 4;
constexpr int kMaxChunks = 64; // a head's partials in the workspace
constexpr int kSub = 16;       // keys per slice (one k16 step of P V)

// bf16: per warp two slots of [K|V][16][D] bf16.  fp8: one f16 slot plus two
// staging slots of raw bytes -- the same 16 KB per warp.
template <int D>
constexpr size_t decode_smem_bytes() { return (size_t)kWarps * 2 * 2 * kSub * D * 2; }

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
template <bool F16>
__device__ __forceinline__ void mma_k16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    mma16816(c, a, b0, b1);
  }
}

template <int D, int REP, bool F8>
__global__ void __launch_bounds__(128) attn_decode_kernel(const DecodeAttnParams p) {
  constexpr int NK = D / 16;   // k16 steps of Q K^T
  constexpr int ND = D / 8;    // 8-dim n-tiles of P V
  constexpr int CPR = D / 8;   // 16-byte chunks per K / V row
  static_assert(REP <= 8, "query heads per kv head fill the upper half of A at most");
  griddep_begin();
  extern __shared__ __align__(128) uint8_t dsm[];
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  const int gid = lane >> 2, tig = lane & 3;
  // A position outside the cache (already reported by the conv kernel) gives
  // an empty key range, so nothing outside the cache is read.
  const int t_raw = p.cache_len[b];
  const int t = (t_raw >= 0 && (p.ring || t_raw < p.cap)) ? t_raw : -1;
  const int lo = max(0, t - p.window + 1);
  const int c_begin = lo + chunk * p.chunk_keys;
  const int c_end = min(t + 1, c_begin + p.chunk_keys);
  const int per_warp = p.chunk_keys / kWarps;
  const int w_begin = c_begin + warp * per_warp;
  const int w_end = min(c_end, w_begin + per_warp);
  // cache row of key w_begin: a window ring keeps position p at slot p % cap;
  // the warp's keys span fewer than cap positions, so they wrap at most once
  const int row0 = p.ring && w_begin < w_end ? w_begin % p.cap : w_begin;
  const float sl2 = p.scale * 1.4426950408889634f;

  // Q fragments: row gid of A is query head g * REP + gid (zero from REP on)
  uint32_t qa[NK][2];
  {
    const auto* qrow = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.n_q + g * REP + gid) * D;
#pragma unroll
    for (int kk = 0; kk < NK; ++kk) {
      qa[kk][0] = gid < REP ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * tig) : 0u;
      qa[kk][1] = gid < REP ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * tig) : 0u;
      if constexpr (F8) {   // the products run in f16
        const float2 x0 = unpack_bf2(qa[kk][0]), x1 = unpack_bf2(qa[kk][1]);
        qa[kk][0] = pack_f16x2(x0.x, x0.y);
        qa[kk][1] = pack_f16x2(x1.x, x1.y);
      }
    }
  }
  constexpr int ES = F8 ? 1 : 2;   // bytes per cached element
  const auto* Kg = static_cast<const uint8_t*>(p.k_cache) + ((size_t)b * p.n_kv + g) * p.cap * D * ES;
  const auto* Vg = static_cast<const uint8_t*>(p.v_cache) + ((size_t)b * p.n_kv + g) * p.cap * D * ES;
  __nv_bfloat16* sw = reinterpret_cast<__nv_bfloat16*>(dsm) + (size_t)warp * 2 * 2 * kSub * D;   // [slot][K|V][16][D]
  // fp8: the f16 slice in slot 0, raw staging slots [2][K|V][16][D] bytes in slot 1's space
  uint8_t* raw = reinterpret_cast<uint8_t*>(sw + 2 * kSub * D);
  // K and V rows key0 .. key0+15 into ring slot `slot` (fp8: staging slot);
  // keys past the warp's range are zero-filled (no global read)
  auto load_slice = [&](int slot, int key0) {
    if constexpr (F8) {
      constexpr int CR = D / 16;   // 16-byte chunks per raw row
      uint8_t* dk = raw + (size_t)slot * 2 * kSub * D;
      uint8_t* dv = dk + kSub * D;
#pragma unroll
      for (int i = lane; i < kSub * CR; i += 32) {
        const int r = i / CR, c = i % CR;
        const int key = key0 + r;
        const bool ok = key < w_end;
        int row = row0 + (key - w_begin);
        if (row >= p.cap) row -= p.cap;
        const size_t src = (size_t)(ok ? row : 0) * D + c * 16;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dk + r * D + c * 16)),
                     "l"(Kg + src), "r"(ok ? 16 : 0)
                     : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dv + r * D + c * 16)),
                     "l"(Vg + src), "r"(ok ? 16 : 0)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      return;
    }
    __nv_bfloat16* dk = sw + (size_t)slot * 2 * kSub * D;
    __nv_bfloat16* dv = dk + kSub * D;
#pragma unroll
    for (int i = lane; i < kSub * CPR; i += 32) {
      const int r = i / CPR, c = i % CPR;
      const int key = key0 + r;
      const bool ok = key < w_end;
      int row = row0 + (key - w_begin);
      if (row >= p.cap) row -= p.cap;
      const size_t src = ((size_t)(ok ? row : 0) * D + c * 8) * 2;
      const int dst = r * D + ((c ^ (r & 7)) * 8);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dk + dst)), "l"(Kg + src),
                   "r"(ok ? 16 : 0)
                   : "memory");
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dv + dst)), "l"(Vg + src),
                   "r"(ok ? 16 : 0)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float m_run = -INFINITY, l_run = 0.f;   // row gid
  float o[ND][4];
#pragma unroll
  for (int j = 0; j < ND; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  const int n_sub = w_end > w_begin ? (w_end - w_begin + kSub - 1) / kSub : 0;
  if (n_sub > 0) load_slice(0, w_begin);
  const int mi = lane >> 3, rr = lane & 7;
  for (int si = 0; si < n_sub; ++si) {
    const int slot = si & 1;
    if (si + 1 < n_sub) {
      load_slice(slot ^ 1, w_begin + (si + 1) * kSub);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    if constexpr (F8) {   // the staged E4M3 slice, K rows then V rows, as f16 into slot 0
      constexpr int CR = D / 16;
      const uint8_t* rk = raw + (size_t)slot * 2 * kSub * D;
#pragma unroll 2
      for (int i = lane; i < 2 * kSub * CR; i += 32) {
        const int kv = i / (kSub * CR), rem = i % (kSub * CR);
        const int r = rem / CR, c = rem % CR;
        const uint4 x = *reinterpret_cast<const uint4*>(rk + kv * kSub * D + r * D + c * 16);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t h[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          h[2 * j] = e4m3x2_to_f16x2((uint16_t)(w[j] & 0xffffu));
          h[2 * j + 1] = e4m3x2_to_f16x2((uint16_t)(w[j] >> 16));
        }
        __nv_bfloat16* dst = sw + kv * kSub * D + r * D;
        *reinterpret_cast<uint4*>(dst + (((2 * c) ^ (r & 7)) * 8)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(dst + (((2 * c + 1) ^ (r & 7)) * 8)) = make_uint4(h[4], h[5], h[6], h[7]);
      }
      __syncwarp();
    }
    const __nv_bfloat16* sK = F8 ? sw : sw + (size_t)slot * 2 * kSub * D;
    const __nv_bfloat16* sV = sK + kSub * D;
    // S = Q K^T over the slice's 16 keys (two 8-key n-tiles)
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int key_r = (mi >> 1) * 8 + rr;   // matrices: keys 0-7 / 8-15 x dims lo / hi of the k16 step
#pragma unroll
      for (int kk = 0; kk < NK; ++kk) {
        const int ch = 2 * kk + (mi & 1);
        uint32_t b00, b01, b10, b11;
        ldsm_x4(smem_u32(sK + key_r * D + ((ch ^ (key_r & 7)) * 8)), b00, b01, b10, b11);
        const uint32_t a[4] = {qa[kk][0], 0u, qa[kk][1], 0u};
        mma_k16<F8>(s[0], a, b00, b01);
        mma_k16<F8>(s[1], a, b10, b11);
      }
    }
    // online softmax on row gid: keys 2tig, 2tig+1 (tile 0) and 8+2tig, 9+2tig (tile 1)
    const int key0 = w_begin + si * kSub;
    float v[4] = {s[0][0], s[0][1], s[1][0], s[1][1]};
    const int kid[4] = {2 * tig, 2 * tig + 1, 8 + 2 * tig, 9 + 2 * tig};
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = (key0 + kid[i] < w_end) ? v[i] * sl2 : -INFINITY;
    float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float base = (m_new == -INFINITY) ? 0.f : m_new;
    const float corr = exp2f(m_run - base);
    float pv[4], ps = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      pv[i] = exp2f(v[i] - base);
      ps += pv[i];
    }
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    l_run = l_run * corr + ps;
    m_run = m_new;
#pragma unroll
    for (int j = 0; j < ND; ++j) {
      o[j][0] *= corr;
      o[j][1] *= corr;
    }
    // O += P V: P (bf16) is the A operand, V read transposed
    const uint32_t pa[4] = {F8 ? pack_f16x2(pv[0], pv[1]) : pack_bf2(pv[0], pv[1]), 0u,
                            F8 ? pack_f16x2(pv[2], pv[3]) : pack_bf2(pv[2], pv[3]), 0u};
    {
      const int key_r = (mi & 1) * 8 + rr;   // matrices: keys 0-7 / 8-15 x dims of n-tiles j / j+1
#pragma unroll
      for (int j = 0; j < ND; j += 2) {
        const int ch = j + (mi >> 1);
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(smem_u32(sV + key_r * D + ((ch ^ (key_r & 7)) * 8)), r0, r1, r2, r3);
        mma_k16<F8>(o[j], pa, r0, r1);
        mma_k16<F8>(o[j + 1], pa, r2, r3);
      }
    }
    __syncwarp();   // the slot is read before the next iteration refills it
  }

  // merge the 4 warps of this CTA (the K / V ring is free now), then write the
  // chunk's partial result
  __syncthreads();
  float* sm_o = reinterpret_cast<float*>(dsm);                 // [kWarps][REP][D]
  float* sm_m = sm_o + kWarps * REP * D;                        // [kWarps][REP]
  float* sm_l = sm_m + kWarps * REP;
  if (gid < REP) {
    if (tig == 0) {
      sm_m[warp * REP + gid] = m_run;
      sm_l[warp * REP + gid] = l_run;
    }
#pragma unroll
    for (int j = 0; j < ND; ++j)
      *reinterpret_cast<float2*>(sm_o + (warp * REP + gid) * D + 8 * j + 2 * tig) = make_float2(o[j][0], o[j][1]);
  }
  __syncthreads();
  const size_t part_idx = (((size_t)b * p.n_kv + g) * p.n_chunks + chunk) * REP;
  float* pm = p.part;                                           // [.., REP] max
  float* pl = p.part + (size_t)p.B * p.n_kv * p.n_chunks * REP; // [.., REP] sum
  float* po = pl + (size_t)p.B * p.n_kv * p.n_chunks * REP;     // [.., REP, D]
  for (int idx = threadIdx.x; idx < REP * D; idx += blockDim.x) {
    const int hh = idx / D, dd = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w * REP + hh]);
    const float bse = (M == -INFINITY) ? 0.f : M;
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = exp2f(sm_m[w * REP + hh] - bse);
      L += sm_l[w * REP + hh] * f;
      O += sm_o[(w * REP + hh) * D + dd] * f;
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
#define ZAYA_DEC(DV, RV, F8V)                                                                          \
  if (p.d == DV && rep == RV && (p.fp8 != 0) == F8V) {                                                 \
    static bool set = false;                                                                           \
    if (!set) {                                                                                        \
      if (cudaFuncSetAttribute(attn_decode_kernel<DV, RV, F8V>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                               (int)decode_smem_bytes<DV>()) != cudaSuccess)                          \
        return ZAYA_ERR_CUDA;                                                                          \
      set = true;                                                                                      \
    }                                                                                                  \
    launch_k(attn_decode_kernel<DV, RV, F8V>, grid, dim3(32 * kWarps), decode_smem_bytes<DV>(), st, nullptr, 0, p); \
    launch_k(attn_decode_combine<DV>, dim3(p.B * p.n_q), dim3(DV), 0, st, nullptr, 0, p, RV);         \
    return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;                                \
  }
#define ZAYA_DEC2(DV, RV) ZAYA_DEC(DV, RV, false) ZAYA_DEC(DV, RV, true)
  ZAYA_DEC2(128, 4)
  ZAYA_DEC2(64, 4)
  ZAYA_DEC2(128, 2)
  ZAYA_DEC2(64, 2)
  ZAYA_DEC2(128, 1)
  ZAYA_DEC2(64, 1)
  ZAYA_DEC2(128, 8)
  ZAYA_DEC2(64, 8)
#undef ZAYA_DEC2
#undef ZAYA_DEC
  return ZAYA_ERR_UNSUPPORTED;
}

}  // namespace zaya
