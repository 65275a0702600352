// Sliding-window causal GQA attention, prefill (flash-attention style).
//
// softmax(q k^T * scale + mask) v for every query head h with kv head
// h / (n_q / n_kv); key j is visible to query i iff 0 <= i - j < window and
// key j is not padding (nnterp "zaya" page: GQA, eager softmax attention;
// window per the workload).  A query with no visible key outputs 0.
//
// CTA = 64 queries of one (sequence, head); 4 warps of 16 query rows.  K/V
// tiles of 64 keys stream through a double-buffered cp.async ring (XOR
// swizzled rows), S = Q K^T and O += P V run on mma.sync m16n8k16 (bf16 in,
// fp32 accumulate), the softmax is online in the exp2 domain.  Only key
// tiles inside the window are visited; masks are applied on tiles that
// straddle the causal diagonal, the window edge, or a padding mask.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

constexpr int kBM = 64;
constexpr int kBN = 64;

template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * D * 2 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 64 rows x D bf16 from global (rows >= limit zero-filled) into swizzled smem.
template <int D>
__device__ __forceinline__ void load_rows(uint32_t sbase, const __nv_bfloat16* g, int row0, int limit) {
  constexpr int CH = D / 8;
  for (int i = threadIdx.x; i < kBM * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    const bool valid = row0 + r < limit;
    const __nv_bfloat16* src = g + (size_t)(valid ? row0 + r : row0) * D + c * 8;
    cp_async16(sbase + swz<D>(r, c), src, valid);
  }
}

template <int D>
__global__ void __launch_bounds__(128) attn_prefill_kernel(const AttnParams p) {
  constexpr int NT = kBN / 8;   // key n-tiles per K tile
  constexpr int DT = D / 8;     // d n-tiles of O
  constexpr int KK = D / 16;    // k-steps of Q K^T
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK0 = sQ + kBM * D * 2;
  const uint32_t sV0 = sK0 + 2 * kBN * D * 2;

  const int qb = gridDim.x - 1 - blockIdx.x;  // heaviest (latest) query blocks first
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (p.n_q / p.n_kv);
  const int m0 = qb * kBM;
  const int warp = warp_id(), lane = lane_id();
  const int S = p.S;

  const auto* Qg = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.n_q + h) * S * D;
  const auto* Kg = static_cast<const __nv_bfloat16*>(p.k_cache) + ((size_t)b * p.n_kv + g) * p.cap * D;
  const auto* Vg = static_cast<const __nv_bfloat16*>(p.v_cache) + ((size_t)b * p.n_kv + g) * p.cap * D;
  const int* mask = p.mask ? p.mask + (size_t)b * S : nullptr;

  const int q_last = min(S, m0 + kBM) - 1;
  const int lo = max(0, m0 - p.window + 1);
  const int n_begin = (lo / kBN) * kBN;
  const int n_end = q_last + 1;  // exclusive
  const int n_tiles = (n_end - n_begin + kBN - 1) / kBN;

  load_rows<D>(sQ, Qg, m0, S);
  if (n_tiles > 0) {
    load_rows<D>(sK0, Kg, n_begin, S);
    load_rows<D>(sV0, Vg, n_begin, S);
  }
  cp_async_commit();

  const float sl2 = p.scale * 1.4426950408889634f;
  const int r_lo = m0 + warp * 16 + (lane >> 2);
  const int r_hi = r_lo + 8;
  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  uint32_t qa[KK][4];

  for (int it = 0; it < n_tiles; ++it) {
    const int buf = it & 1;
    const int n0 = n_begin + it * kBN;
    cp_async_wait_all();
    __syncthreads();
    if (it == 0) {
#pragma unroll
      for (int kk = 0; kk < KK; ++kk)
        ldsm_x4(sQ + swz<D>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), qa[kk][0], qa[kk][1], qa[kk][2],
                qa[kk][3]);
    }
    if (it + 1 < n_tiles) {  // prefetch the next tile into the other buffer
      load_rows<D>(sK0 + (buf ^ 1) * kBN * D * 2, Kg, n0 + kBN, S);
      load_rows<D>(sV0 + (buf ^ 1) * kBN * D * 2, Vg, n0 + kBN, S);
    }
    cp_async_commit();
    const uint32_t sK = sK0 + buf * kBN * D * 2;
    const uint32_t sV = sV0 + buf * kBN * D * 2;

    float s[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
#pragma unroll
      for (int kk = 0; kk < KK; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz<D>(np * 16 + ((lane >> 4) << 3) + (lane & 7), kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma16816(s[2 * np], qa[kk], b0, b1);
        mma16816(s[2 * np + 1], qa[kk], b2, b3);
      }
    }

    const bool need_mask = mask != nullptr || (n0 + kBN - 1 > m0) || (m0 + kBM - 1 - n0 >= p.window) ||
                           (n0 + kBN > S);
    float tmax_lo = -INFINITY, tmax_hi = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = n0 + nt * 8 + (lane & 3) * 2 + (e & 1);
        const int row = (e < 2) ? r_lo : r_hi;
        float v = s[nt][e] * sl2;
        if (need_mask) {
          const bool vis = key <= row && row - key < p.window && key < S && (!mask || mask[key] != 0);
          if (!vis) v = -INFINITY;
        }
        s[nt][e] = v;
      }
      tmax_lo = fmaxf(tmax_lo, fmaxf(s[nt][0], s[nt][1]));
      tmax_hi = fmaxf(tmax_hi, fmaxf(s[nt][2], s[nt][3]));
    }
    tmax_lo = fmaxf(tmax_lo, __shfl_xor_sync(0xffffffffu, tmax_lo, 1));
    tmax_lo = fmaxf(tmax_lo, __shfl_xor_sync(0xffffffffu, tmax_lo, 2));
    tmax_hi = fmaxf(tmax_hi, __shfl_xor_sync(0xffffffffu, tmax_hi, 1));
    tmax_hi = fmaxf(tmax_hi, __shfl_xor_sync(0xffffffffu, tmax_hi, 2));
    const float mn_lo = fmaxf(m_lo, tmax_lo), mn_hi = fmaxf(m_hi, tmax_hi);
    const float base_lo = (mn_lo == -INFINITY) ? 0.f : mn_lo;
    const float base_hi = (mn_hi == -INFINITY) ? 0.f : mn_hi;
    const float corr_lo = exp2f(m_lo - base_lo), corr_hi = exp2f(m_hi - base_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    float ps_lo = 0.f, ps_hi = 0.f;
    uint32_t pa[NT / 2][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float p0 = exp2f(s[nt][0] - base_lo), p1 = exp2f(s[nt][1] - base_lo);
      const float p2 = exp2f(s[nt][2] - base_hi), p3 = exp2f(s[nt][3] - base_hi);
      ps_lo += p0 + p1;
      ps_hi += p2 + p3;
      pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf2(p0, p1);
      pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf2(p2, p3);
    }
    l_lo = l_lo * corr_lo + ps_lo;
    l_hi = l_hi * corr_hi + ps_hi;
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      o[i][0] *= corr_lo;
      o[i][1] *= corr_lo;
      o[i][2] *= corr_hi;
      o[i][3] *= corr_hi;
    }
#pragma unroll
    for (int kk = 0; kk < NT / 2; ++kk) {
      // A fragment order: (row lo, keys 0-7), (row hi, keys 0-7), (row lo, keys 8-15), (row hi, keys 8-15)
      const uint32_t a[4] = {pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3]};
#pragma unroll
      for (int dp = 0; dp < DT / 2; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + swz<D>(kk * 16 + (((lane >> 3) & 1) << 3) + (lane & 7), dp * 2 + (lane >> 4)), b0, b1, b2,
                  b3);
        mma16816(o[2 * dp], a, b0, b1);
        mma16816(o[2 * dp + 1], a, b2, b3);
      }
    }
  }

  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
  const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f;
  const float inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
  const int ld = p.n_q * D;
  auto* out = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll
  for (int i = 0; i < DT; ++i) {
    const int col = h * D + i * 8 + (lane & 3) * 2;
    if (r_lo < S)
      *reinterpret_cast<uint32_t*>(out + ((size_t)b * S + r_lo) * ld + col) = pack_bf2(o[i][0] * inv_lo, o[i][1] * inv_lo);
    if (r_hi < S)
      *reinterpret_cast<uint32_t*>(out + ((size_t)b * S + r_hi) * ld + col) = pack_bf2(o[i][2] * inv_hi, o[i][3] * inv_hi);
  }
}

}  // namespace

int launch_attn_prefill(const AttnParams& p, cudaStream_t st) {
  if (p.B <= 0 || p.S <= 0) return ZAYA_OK;
  const dim3 grid((p.S + kBM - 1) / kBM, p.n_q, p.B);
  if (p.d == 128) {
    const int smem = 5 * kBM * 128 * 2;
    static bool set = false;
    if (!set) {
      cudaFuncSetAttribute(attn_prefill_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      set = true;
    }
    attn_prefill_kernel<128><<<grid, 128, smem, st>>>(p);
  } else if (p.d == 64) {
    const int smem = 5 * kBM * 64 * 2;
    attn_prefill_kernel<64><<<grid, 128, smem, st>>>(p);
  } else {
    return ZAYA_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

}  // namespace zaya
