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
  constexpr int NT = 2 * D;       // threads
  constexpr int VPR = D / 8;      // 16-byte vectors of u per row
  griddep_begin();
  extern __shared__ __align__(16) uint32_t sw[];
  uint32_t* Ws = sw;                                   // [D outputs][LDS] TF32
  uint32_t* As = sw + (size_t)D * LDS;                 // [kTileTok tokens][LDS] TF32
  __nv_bfloat16* Us = reinterpret_cast<__nv_bfloat16*>(As + (size_t)kTileTok * LDS);   // [kTileTok + 2][D]
  const int g = blockIdx.y;
  const int C = p.C;
  const int warp = warp_id(), lane = lane_id();
  const int gid = lane >> 2, tig = lane & 3;
  const auto* qkv = static_cast<const __nv_bfloat16*>(p.qkv);

  // the group's weights, [out][tap * D + in] (global layout [C][D][2], Conv1d's):
  // four consecutive words are (in, tap 0), (in, tap 1), (in+1, tap 0), (in+1, tap 1)
  {
    const float4* gw4 = reinterpret_cast<const float4*>(p.gw + (size_t)g * D * K);
    constexpr int N4 = D * K / 4, PER = N4 / NT;
#pragma unroll 8
    for (int j = 0; j < PER; ++j) {
      const int e4 = threadIdx.x + j * NT;
      const float4 v = __ldg(gw4 + e4);
      const int o = (4 * e4) / K, i = ((4 * e4) % K) >> 1;
      uint32_t* w = Ws + o * LDS + i;
      w[0] = to_tf32(v.x);
      w[D] = to_tf32(v.y);
      w[1] = to_tf32(v.z);
      w[D + 1] = to_tf32(v.w);
    }
  }
  // this thread's channel pair: depthwise taps and bias, loaded once
  const int cp = threadIdx.x % (D / 2), rsub = threadIdx.x / (D / 2);   // NT / (D/2) = 4 row lanes
  const int c0 = g * D + 2 * cp;
  const float4 dwv = __ldg(reinterpret_cast<const float4*>(p.dw + 2 * c0));   // (c0: t-1, t), (c0+1: t-1, t)
  const float2 dbv = __ldg(reinterpret_cast<const float2*>(p.db + c0));
  const int n_tiles = (p.rows + kTileTok - 1) / kTileTok;

  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    __syncthreads();   // the previous tile's rows are consumed
    const int m0 = tile * kTileTok;
    if (!p.decode) {
      // u rows m0-2 .. m0+63 of the group's channels (zero before a sequence, past the
      // end and at padding), one cp.async wait
      for (int v = threadIdx.x; v < (kTileTok + 2) * VPR; v += NT) {
        const int r = v / VPR, c8 = v % VPR;
        const int m = m0 - 2 + r;
        const int mm = m < 0 ? 0 : (m >= p.rows ? p.rows - 1 : m);
        // rows outside [0, rows) and padding rows are zero; rows of a previous
        // sequence are loaded but not used (the z rows below test the position)
        const bool ok = m >= 0 && m < p.rows && (!p.mask || p.mask[mm] != 0);
        const __nv_bfloat16* src = qkv + (size_t)mm * p.ld + g * D + c8 * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(Us + (size_t)r * D + c8 * 8)),
                     "l"(src), "r"(ok ? 16 : 0)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncthreads();
    }
    // [z(t-1) || z(t)] rows: thread = (row lane, channel pair)
    for (int r = rsub; r < kTileTok; r += NT / (D / 2)) {
      const int m = m0 + r;
      float2 u0 = make_float2(0.f, 0.f), u1 = u0, u2 = u0;   // u[t], u[t-1], u[t-2]
      if (m < p.rows) {
        if (p.decode) {
          const auto* cs = static_cast<const __nv_bfloat16*>(p.conv_state) + ((size_t)m * C + c0) * 2;
          u0 = unpack_bf2(*reinterpret_cast<const uint32_t*>(qkv + (size_t)m * p.ld + c0));
          const float2 s0 = unpack_bf2(*reinterpret_cast<const uint32_t*>(cs));       // c0: t-2, t-1
          const float2 s1 = unpack_bf2(*reinterpret_cast<const uint32_t*>(cs + 2));   // c0+1: t-2, t-1
          u2 = make_float2(s0.x, s1.x);
          u1 = make_float2(s0.y, s1.y);
        } else {
          const int s = m % p.S;
          u0 = unpack_bf2(*reinterpret_cast<const uint32_t*>(Us + (size_t)(r + 2) * D + 2 * cp));
          if (s >= 1) u1 = unpack_bf2(*reinterpret_cast<const uint32_t*>(Us + (size_t)(r + 1) * D + 2 * cp));
          if (s >= 2) u2 = unpack_bf2(*reinterpret_cast<const uint32_t*>(Us + (size_t)r * D + 2 * cp));
        }
      }
      uint32_t* a = As + r * LDS + 2 * cp;
      a[0] = to_tf32(fmaf(dwv.x, u2.x, fmaf(dwv.y, u1.x, dbv.x)));       // z(t-1), c0
      a[1] = to_tf32(fmaf(dwv.z, u2.y, fmaf(dwv.w, u1.y, dbv.y)));       // z(t-1), c0+1
      a[D] = to_tf32(fmaf(dwv.x, u1.x, fmaf(dwv.y, u0.x, dbv.x)));       // z(t), c0
      a[D + 1] = to_tf32(fmaf(dwv.z, u1.y, fmaf(dwv.w, u0.y, dbv.y)));   // z(t), c0+1
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
      const int m_lo = m0 + r0 + gid, m_hi = m_lo + 8;
      if (m_lo < p.rows)
        *reinterpret_cast<float2*>(p.y + (size_t)m_lo * C + o) = make_float2(acc[j][0] + b0, acc[j][1] + b1);
      if (m_hi < p.rows)
        *reinterpret_cast<float2*>(p.y + (size_t)m_hi * C + o) = make_float2(acc[j][2] + b0, acc[j][3] + b1);
    }
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
  const size_t smem = (size_t)(d + kTileTok) * (2 * d + 4) * 4 + (size_t)(kTileTok + 2) * d * 2;
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
