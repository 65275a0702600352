// The pages' two-stage conv_qk (nnterp "zaya" page, "Printout": conv_qk_depthwise
// Conv1d(C, C, k=2, groups=C), then conv_qk_grouped Conv1d(C, C, k=2, groups=G);
// "Queries and keys are convolved ...": the current and two previous tokens):
//
//   z[s, c] = dw[c, 0] u[s-1, c] + dw[c, 1] u[s, c] + db[c]
//   y[t, o] = sum_i gw[o, i, 0] z[t-1, g(o) D + i] + gw[o, i, 1] z[t, g(o) D + i] + gb[o]
//
// with one group per q / k head (G = n_q + n_kv, D = head_dim channels each).
// u is the pre-conv q||k projection (bf16), zero before the sequence and at
// padding in prefill; in decode u[t-2], u[t-1] come from conv_state.  The
// grouped stage is a [tokens, 2D] x [2D, D] product per group on the tensor
// cores in TF32 (mma.sync m16n8k8, fp32 accumulation): z is fp32, the conv
// weights are kept in float by the deployments, and TF32's 10-bit mantissa
// keeps the product's error near the bf16 rounding the q / k heads get later.
// Output y fp32 [rows, C], read by the CCA kernel in place of its width-3 conv.
//
// CTA = one group, persistent over 64-token tiles: the group's weights
// (D x 2D, converted to TF32 once) and a tile's [z(t-1) || z(t)] rows sit in
// shared memory with rows padded by 4 words, so every fragment load is free
// of bank conflicts; warp w computes 16 tokens x 64 outputs.
#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

constexpr int kTileTok = 64;

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// C[16x8] += A[16x8] * B[8x8], TF32 in, fp32 accumulate.
__device__ __forceinline__ void mma_tf32(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(2 * D) conv_grouped_kernel(const ConvGroupedParams p) {
  constexpr int K = 2 * D;        // [z(t-1) || z(t)]
  constexpr int LDS = K + 4;      // padded row (words)
  constexpr int NH = D / 64;      // 64-output halves
  griddep_begin();
  extern __shared__ __align__(16) uint32_t sw[];
  uint32_t* Ws = sw;                         // [D outputs][LDS] TF32
  uint32_t* As = sw + (size_t)D * LDS;       // [kTileTok tokens][LDS] TF32
  const int g = blockIdx.y;
  const int C = p.C;
  const int warp = warp_id(), lane = lane_id();
  const int gid = lane >> 2, tig = lane & 3;

  // the group's weights, [out][tap * D + in] (global layout [C][D][2], Conv1d's)
  const float* gw = p.gw + (size_t)g * D * K;
  for (int e = threadIdx.x; e < D * K; e += blockDim.x) {
    const int o = e / K, rem = e % K, i = rem >> 1, tap = rem & 1;
    Ws[o * LDS + tap * D + i] = to_tf32(__ldg(gw + e));
  }
  const auto* qkv = static_cast<const __nv_bfloat16*>(p.qkv);
  const auto* cstate = static_cast<const __nv_bfloat16*>(p.conv_state);
  const int n_tiles = (p.rows + kTileTok - 1) / kTileTok;

  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    __syncthreads();   // the weights are in; the previous tile's rows are consumed
    // [z(t-1) || z(t)] of the tile's tokens for the group's D channels
    for (int e = threadIdx.x; e < kTileTok * D; e += blockDim.x) {
      const int r = e / D, i = e % D, c = g * D + i;
      const int m = tile * kTileTok + r;
      float u0 = 0.f, u1 = 0.f, u2 = 0.f;   // u[t], u[t-1], u[t-2]
      if (m < p.rows) {
        if (p.decode) {
          u0 = bf2f(qkv[(size_t)m * p.ld + c]);
          u1 = bf2f(cstate[((size_t)m * C + c) * 2 + 1]);
          u2 = bf2f(cstate[((size_t)m * C + c) * 2 + 0]);
        } else {
          const int s = m % p.S;
          const int* mk = p.mask ? p.mask + (m - s) : nullptr;
          if (!mk || mk[s]) u0 = bf2f(qkv[(size_t)m * p.ld + c]);
          if (s >= 1 && (!mk || mk[s - 1])) u1 = bf2f(qkv[(size_t)(m - 1) * p.ld + c]);
          if (s >= 2 && (!mk || mk[s - 2])) u2 = bf2f(qkv[(size_t)(m - 2) * p.ld + c]);
        }
      }
      const float d0 = __ldg(p.dw + 2 * c), d1 = __ldg(p.dw + 2 * c + 1), bb = __ldg(p.db + c);
      As[r * LDS + i] = to_tf32(fmaf(d0, u2, fmaf(d1, u1, bb)));        // z(t-1)
      As[r * LDS + D + i] = to_tf32(fmaf(d0, u1, fmaf(d1, u0, bb)));    // z(t)
    }
    __syncthreads();
    const int r0 = (warp & 3) * 16;
    const int n0 = (warp >> 2) * 64;
    float acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll 4
    for (int k0 = 0; k0 < K; k0 += 8) {
      const uint32_t a0 = As[(r0 + gid) * LDS + k0 + tig];
      const uint32_t a1 = As[(r0 + gid + 8) * LDS + k0 + tig];
      const uint32_t a2 = As[(r0 + gid) * LDS + k0 + tig + 4];
      const uint32_t a3 = As[(r0 + gid + 8) * LDS + k0 + tig + 4];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t* wr = Ws + (n0 + 8 * j + gid) * LDS + k0 + tig;
        mma_tf32(acc[j], a0, a1, a2, a3, wr[0], wr[4]);
      }
    }
    // y rows of the tile: the warp's 16 tokens x 64 outputs, plus the bias
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int o = g * D + n0 + 8 * j + 2 * tig;
      const float b0 = __ldg(p.gb + o), b1 = __ldg(p.gb + o + 1);
      const int m_lo = tile * kTileTok + r0 + gid, m_hi = m_lo + 8;
      if (m_lo < p.rows)
        *reinterpret_cast<float2*>(p.y + (size_t)m_lo * C + o) = make_float2(acc[j][0] + b0, acc[j][1] + b1);
      if (m_hi < p.rows)
        *reinterpret_cast<float2*>(p.y + (size_t)m_hi * C + o) = make_float2(acc[j][2] + b0, acc[j][3] + b1);
    }
    (void)NH;
  }
}

}  // namespace

int launch_conv_grouped(const ConvGroupedParams& p, int groups, int d, int num_sms, cudaStream_t st) {
  if (p.rows <= 0) return ZAYA_OK;
  if (d != 64 && d != 128) return ZAYA_ERR_UNSUPPORTED;
  const int n_tiles = (p.rows + kTileTok - 1) / kTileTok;
  int per_group = num_sms / groups;
  if (per_group < 1) per_group = 1;
  if (per_group > n_tiles) per_group = n_tiles;
  const dim3 grid(per_group, groups);
  const size_t smem = (size_t)(d + kTileTok) * (2 * d + 4) * 4;
  if (d == 128) {
    cudaFuncSetAttribute(conv_grouped_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_k(conv_grouped_kernel<128>, grid, dim3(256), smem, st, nullptr, 0, p);
  } else {
    cudaFuncSetAttribute(conv_grouped_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_k(conv_grouped_kernel<64>, grid, dim3(128), smem, st, nullptr, 0, p);
  }
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

}  // namespace zaya
