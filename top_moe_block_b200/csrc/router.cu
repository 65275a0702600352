// Router MLP, scoring and top-1 choice with the skip class; the stable
// token -> expert permutation; the dispatch of routed rows and the merge of
// skipped rows.
//
// Router (nnterp "zaya" page, "One expert per token, chosen beside a skip
// class", and the ZayaRouterMLP printout): router_logits =
// out_proj(gelu(fc2(gelu(fc1(rmsnorm(r)))))) over E + 1 classes, the last
// being skip; p = softmax(logits) in fp32; class = argmax(p +
// balancing_biases), the lowest index on exact ties; weight = p[class] (not
// renormalised); skip -> (index 0, weight 0).  Runs in fp32 on CUDA cores:
// 16 tokens per CTA, each 256x256 layer as a register-tiled product whose
// weight slab is staged transposed in shared memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

constexpr int kTM = 16;     // tokens per router CTA
constexpr int kKC = 32;     // k-chunk of a weight slab
constexpr int kRMax = 256;

__device__ __forceinline__ float gelu_exact(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

// out[tt][j] = gelu(sum_k in[tt][k] * W[j][k] + bias[j]) for tt < kTM, j < R.
__device__ __forceinline__ void dense_gelu(const float* __restrict__ in, float* __restrict__ out,
                                           const float* __restrict__ W, const float* __restrict__ bias, float* wt,
                                           int R) {
  const int j = threadIdx.x;
  float acc[kTM];
#pragma unroll
  for (int t = 0; t < kTM; ++t) acc[t] = 0.f;
  for (int kc = 0; kc < R; kc += kKC) {
    __syncthreads();
    for (int i = threadIdx.x; i < R * kKC; i += blockDim.x) {
      const int jj = i / kKC, k = i % kKC;
      wt[k * (kRMax + 1) + jj] = __ldg(W + (size_t)jj * R + kc + k);
    }
    __syncthreads();
    if (j < R) {
#pragma unroll 4
      for (int k = 0; k < kKC; k += 4) {
        const float w0 = wt[(k + 0) * (kRMax + 1) + j], w1 = wt[(k + 1) * (kRMax + 1) + j];
        const float w2 = wt[(k + 2) * (kRMax + 1) + j], w3 = wt[(k + 3) * (kRMax + 1) + j];
#pragma unroll
        for (int t = 0; t < kTM; ++t) {
          const float4 x = *reinterpret_cast<const float4*>(in + t * kRMax + kc + k);
          acc[t] = fmaf(x.x, w0, fmaf(x.y, w1, fmaf(x.z, w2, fmaf(x.w, w3, acc[t]))));
        }
      }
    }
  }
  if (j < R) {
    const float bj = __ldg(bias + j);
#pragma unroll
    for (int t = 0; t < kTM; ++t) out[t * kRMax + j] = gelu_exact(acc[t] + bj);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256) router_kernel(const RouterParams p) {
  extern __shared__ __align__(16) float sm[];
  float* z = sm;                         // [kTM][kRMax]
  float* g = z + kTM * kRMax;            // [kTM][kRMax]
  float* wt = g + kTM * kRMax;           // [kKC][kRMax + 1]
  float* lg = wt + kKC * (kRMax + 1);    // [kTM][E+1]
  const int R = p.R, E1 = p.E + 1;
  const int t0 = blockIdx.x * kTM;
  const int warp = warp_id(), lane = lane_id();

  for (int i = threadIdx.x; i < kTM * R; i += blockDim.x) {
    const int tt = i / R, k = i % R;
    z[tt * kRMax + k] = (t0 + tt < p.M) ? p.r[(size_t)(t0 + tt) * R + k] : 0.f;
  }
  __syncthreads();
  for (int tt = warp; tt < kTM; tt += 8) {   // router_mlp.norm (RMSNorm over R)
    float ss = 0.f;
    for (int k = lane; k < R; k += 32) ss += z[tt * kRMax + k] * z[tt * kRMax + k];
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / (float)R + p.eps);
    for (int k = lane; k < R; k += 32) z[tt * kRMax + k] = __ldg(p.norm_w + k) * (z[tt * kRMax + k] * inv);
  }
  dense_gelu(z, g, p.fc1_w, p.fc1_b, wt, R);
  dense_gelu(g, z, p.fc2_w, p.fc2_b, wt, R);
  for (int i = threadIdx.x; i < kTM * E1; i += blockDim.x) {   // out_proj (no bias)
    const int tt = i / E1, c = i % E1;
    const float* wr = p.out_w + (size_t)c * R;
    float a = 0.f;
    for (int k = 0; k < R; k += 4) {
      const float4 w4 = __ldg(reinterpret_cast<const float4*>(wr + k));
      const float4 x4 = *reinterpret_cast<const float4*>(z + tt * kRMax + k);
      a = fmaf(x4.x, w4.x, fmaf(x4.y, w4.y, fmaf(x4.z, w4.z, fmaf(x4.w, w4.w, a))));
    }
    lg[tt * E1 + c] = a;
  }
  __syncthreads();
  for (int tt = warp; tt < kTM; tt += 8) {   // softmax, balancing, top-1, skip
    const int t = t0 + tt;
    if (t >= p.M) continue;
    float l[3], s[3], e[3];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int c = lane + 32 * u;
      l[u] = c < E1 ? lg[tt * E1 + c] : -INFINITY;
      mx = fmaxf(mx, l[u]);
    }
    mx = warp_max(mx);
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      e[u] = (lane + 32 * u < E1) ? expf(l[u] - mx) : 0.f;
      sum += e[u];
    }
    sum = warp_sum(sum);
    float best = -INFINITY, bestp = 0.f;
    int bc = 0x7fffffff;
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int c = lane + 32 * u;
      if (c < E1) {
        const float pc = e[u] / sum;
        s[u] = pc + __ldg(p.balancing + c);
        if (s[u] > best) {
          best = s[u];
          bc = c;
          bestp = pc;
        }
        p.logits[(size_t)t * E1 + c] = l[u];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
      const float op = __shfl_xor_sync(0xffffffffu, bestp, o);
      if (ob > best || (ob == best && oc < bc)) {
        best = ob;
        bc = oc;
        bestp = op;
      }
    }
    if (lane == 0) {
      int cls = bc;
      if (p.mask && p.mask[t] == 0) cls = p.E;   // padding tokens are routed to skip
      const bool skip = cls == p.E;
      const float w = skip ? 0.f : bestp;
      p.cls[t] = cls;
      p.w[t] = w;
      if (p.idx) p.idx[t] = skip ? 0 : cls;
      if (p.w_tap) p.w_tap[t] = w;
    }
  }
}

// Stable counting sort by class, one CTA of 32 warps; warp w owns a
// contiguous token range, so token order is kept inside every class.
__global__ void __launch_bounds__(1024) permute_kernel(const int* __restrict__ cls, int M, int E, int* group_off,
                                                       int* mt_start, int* pos, int* perm, int* status) {
  __shared__ int cnt[32][66];
  __shared__ int cls_base[66];
  const int warp = warp_id(), lane = lane_id();
  const int E1 = E + 1;
  for (int i = threadIdx.x; i < 32 * 66; i += blockDim.x) cnt[i / 66][i % 66] = 0;
  __syncthreads();
  const int per = ((M + 31) / 32 + 31) / 32 * 32;
  const int begin = warp * per, end = min(M, begin + per);
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = begin; base < end; base += 32) {
    const int t = base + lane;
    int c = -1;
    if (t < end) {
      c = cls[t];
      if (c < 0 || c > E) {
        set_status(status, ZAYA_ERR_DEVICE_RANGE);
        c = E;
      }
    }
    const unsigned same = __match_any_sync(0xffffffffu, c);
    const int rank = __popc(same & lt_mask);
    const int leader = __ffs(same) - 1;
    const int before = (c >= 0) ? cnt[warp][c] : 0;
    __syncwarp();
    if (c >= 0 && lane == leader) cnt[warp][c] = before + __popc(same);
    __syncwarp();
    if (t < end) pos[t] = before + rank;
  }
  __syncthreads();
  // exclusive scan of cnt over (class-major, warp-minor)
  for (int c = warp; c < E1; c += 32) {
    int v = cnt[lane][c];
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += n;
    }
    cnt[lane][c] = inc - v;                              // offset of warp 'lane' inside class c
    if (lane == 31) cls_base[c] = inc;                   // class total (scanned below)
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0, tcarry = 0;
    for (int c0 = 0; c0 < E1; c0 += 32) {
      const int c = c0 + lane;
      const int tot = c < E1 ? cls_base[c] : 0;
      const int tiles = (c < E) ? (tot + 127) / 128 : 0;
      int inc = tot, tinc = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        const int tn = __shfl_up_sync(0xffffffffu, tinc, o);
        if (lane >= o) {
          inc += n;
          tinc += tn;
        }
      }
      __syncwarp();
      if (c < E1) {
        cls_base[c] = carry + inc - tot;
        group_off[c] = carry + inc - tot;
        mt_start[c] = tcarry + tinc - tiles;
      }
      carry += __shfl_sync(0xffffffffu, inc, 31);
      tcarry += __shfl_sync(0xffffffffu, tinc, 31);
      __syncwarp();
    }
    if (lane == 0) {
      mt_start[E1] = tcarry;   // unused entry past the skip class
    }
  }
  __syncthreads();
  for (int base = begin; base < end; base += 32) {
    const int t = base + lane;
    if (t < end) {
      int c = cls[t];
      if (c < 0 || c > E) c = E;
      const int ps = cls_base[c] + cnt[warp][c] + pos[t];
      pos[t] = ps;
      perm[ps] = t;
    }
  }
}

__global__ void __launch_bounds__(256) dispatch_kernel(const DispatchParams p) {
  const int t = blockIdx.x * 8 + warp_id();
  const int lane = lane_id();
  if (t >= p.M) return;
  const int H = p.H;
  const int c = p.cls[t];
  if (c >= 0 && c < p.E) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.m_in) + (size_t)t * H);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.x_perm) + (size_t)p.pos[t] * H);
    for (int i = lane; i < H / 8; i += 32) dst[i] = src[i];
  } else {
    // skip: no expert runs; mlp_output = bf16(hb * hs), out = mlp_output + (h + rb) * rs
    float4* s4 = reinterpret_cast<float4*>(p.stream + (size_t)t * H);
    __nv_bfloat16* tap = p.tap_mlp_out ? static_cast<__nv_bfloat16*>(p.tap_mlp_out) + (size_t)t * H : nullptr;
    for (int i = lane; i < H / 4; i += 32) {
      float4 x = s4[i];
      float* xp = &x.x;
      float cb[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = 4 * i + j;
        const float contrib = round_bf(__ldg(p.merge_m + col) * __ldg(p.merge_m + H + col));
        cb[j] = contrib;
        xp[j] = fmaf(xp[j] + __ldg(p.merge_m + 2 * H + col), __ldg(p.merge_m + 3 * H + col), contrib);
      }
      s4[i] = x;
      if (tap) {
        uint2 u;
        u.x = pack_bf2(cb[0], cb[1]);
        u.y = pack_bf2(cb[2], cb[3]);
        reinterpret_cast<uint2*>(tap)[i] = u;
      }
    }
  }
  if (p.cache_len_inc && lane == 0) p.cache_len_inc[t] += 1;
}

}  // namespace

int launch_router(const RouterParams& p, cudaStream_t st) {
  if (p.M <= 0) return ZAYA_OK;
  if (p.R > kRMax || p.R % 32 || p.E + 1 > 96) return ZAYA_ERR_UNSUPPORTED;
  const size_t smem = sizeof(float) * (2 * kTM * kRMax + kKC * (kRMax + 1) + kTM * (p.E + 1));
  static bool set = false;
  if (!set) {
    cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
    set = true;
  }
  router_kernel<<<(p.M + kTM - 1) / kTM, 256, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

int launch_permute(const int* cls, int M, int E, int* group_off, int* mt_start, int* pos, int* perm, int* status,
                   cudaStream_t st) {
  if (E + 1 > 65) return ZAYA_ERR_UNSUPPORTED;
  permute_kernel<<<1, 1024, 0, st>>>(cls, M, E, group_off, mt_start, pos, perm, status);
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

int launch_dispatch(const DispatchParams& p, cudaStream_t st) {
  if (p.M <= 0) return ZAYA_OK;
  dispatch_kernel<<<(p.M + 7) / 8, 256, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

}  // namespace zaya
