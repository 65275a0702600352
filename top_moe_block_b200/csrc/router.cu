// Router MLP, scoring and top-1 choice with the skip class (each CTA also
// reserves its tokens' places among their class's rows); the token -> expert
// permutation with the dispatch of routed rows and the merge of skipped rows.
//
// Router (nnterp "zaya" page, "One expert per token, chosen beside a skip
// class", and the ZayaRouterMLP printout): router_logits =
// out_proj(gelu(fc2(gelu(fc1(rmsnorm(r)))))) over E + 1 classes, the last
// being skip; p = softmax(logits) in fp32; class = argmax(p +
// balancing_biases), the lowest index on exact ties; weight = p[class] (not
// renormalised); skip -> (index 0, weight 0).  The choice is taken on fp32
// scores, so the logits must carry fp32 accuracy: fc1, fc2 and out_proj run
// on tensor cores with both operands split into bf16 hi + lo parts (three
// products hi.hi + hi.lo + lo.hi, fp32 accumulation: ~16 significant bits per
// product, about fp32's error after the 256-term sums); norm, GELU and the
// softmax run in fp32 on CUDA cores.  32 tokens per CTA; the fc1 / fc2 weight
// chunks arrive by TMA.
#include <math.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

constexpr int kTM = 32;          // tokens per router CTA
constexpr int kThreads = 512;    // 16 warps: warp w -> rows 16*(w&1) .., output group w>>1
constexpr int kRMax = 256;
constexpr int kZS = kRMax + 8;   // row stride (floats) of the fp32 activation tile
constexpr int kAS = kRMax + 8;   // row stride (bf16) of the hi / lo operand tiles: conflict-free ldmatrix

__device__ __forceinline__ float gelu_exact(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

// fp32 -> (hi, lo) bf16 with hi + lo equal to x to about 16 significant bits.
__device__ __forceinline__ void split_bf(float x, float& hi, float& lo) {
  hi = round_bf(x);
  lo = x - hi;
}

template <int R>
struct RouterShape {
  static constexpr int KCH = R < 64 ? R : 64;       // k columns per staged weight chunk
  // R >= 64: chunks arrive by TMA as [R rows][128 bytes] with the 128-byte
  // swizzle (16-byte units XOR row & 7), which keeps ldmatrix conflict-free;
  // R = 32: cp.async into rows padded to KCH + 8
  static constexpr bool TMA = R >= 64;
  static constexpr int WS = TMA ? KCH : KCH + 8;    // bf16 row stride of a chunk
  static constexpr int CHUNK = R * WS;              // bf16 elements of one (hi or lo) chunk
  static constexpr int NG = R / 8 < 8 ? R / 8 : 8;  // output groups (warp pairs)
  static constexpr int NTW = R / (8 * NG);          // 8-wide n-tiles per warp
  static constexpr size_t RING_OFF = sizeof(float) * kTM * kZS + sizeof(__nv_bfloat16) * 2 * kTM * kAS;
  static constexpr size_t SMEM = RING_OFF + sizeof(__nv_bfloat16) * 2 * 2 * CHUNK + (TMA ? 1024 : 0);
};

// Byte offset of bf16 element (row, col) inside a staged weight chunk.
template <int R>
__device__ __forceinline__ uint32_t wofs(int row, int col) {
  using Sh = RouterShape<R>;
  if constexpr (Sh::TMA)
    return (uint32_t)row * 128u + ((uint32_t)((col >> 3) ^ (row & 7)) << 4) + (uint32_t)(col & 7) * 2u;
  else
    return (uint32_t)(row * Sh::WS + col) * 2u;
}

// Stage columns [kc, kc+KCH) of the split weight (hi and lo, [R][R] bf16) into a padded chunk.
template <int R>
__device__ __forceinline__ void stage_chunk(__nv_bfloat16* dst, const __nv_bfloat16* __restrict__ whi,
                                            const __nv_bfloat16* __restrict__ wlo, int kc) {
  using Sh = RouterShape<R>;
  constexpr int V = Sh::KCH / 8;   // 16-byte vectors per row
  for (int i = threadIdx.x; i < 2 * R * V; i += kThreads) {
    const int part = i / (R * V), rem = i % (R * V);
    const int row = rem / V, c = rem % V;
    const __nv_bfloat16* src = (part ? wlo : whi) + (size_t)row * R + kc + c * 8;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst + part * Sh::CHUNK + row * Sh::WS + c * 8)),
                 "l"(src)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// acc[t][j] += sum_{k in chunk c} a[t][k] W[j][k] for the CTA's 32 tokens, on
// tensor cores (mma.sync m16n8k16) with both operands split into bf16 hi + lo:
// a.W ~= a_hi.W_hi + a_hi.W_lo + a_lo.W_hi, fp32 accumulation.  ah / al are the
// activation's hi / lo tiles ([32][kAS]); wh / wl the staged weight chunk.
template <int R, bool LO>   // LO: the weights have lo parts (else wl is not read)
__device__ __forceinline__ void mlp_chunk(const __nv_bfloat16* ah_t, const __nv_bfloat16* al_t, float (*acc)[4],
                                          const __nv_bfloat16* wh, const __nv_bfloat16* wl, int c) {
  using Sh = RouterShape<R>;
  const int warp = warp_id(), lane = lane_id();
  const int rg = warp & 1, ng = warp >> 1;
  if (ng >= Sh::NG) return;
  const int g = lane >> 2, t = lane & 3;
  const int nbase = ng * (R / Sh::NG);
  const int arow = rg * 16 + (lane & 15);
  const int m = lane >> 3;
#pragma unroll
  for (int ks = 0; ks < Sh::KCH / 16; ++ks) {
    const int acol = c * Sh::KCH + ks * 16 + (lane >> 4) * 8;
    uint32_t ah[4], al[4];
    ldsm_x4(smem_u32(ah_t + arow * kAS + acol), ah[0], ah[1], ah[2], ah[3]);
    ldsm_x4(smem_u32(al_t + arow * kAS + acol), al[0], al[1], al[2], al[3]);
#pragma unroll
    for (int j = 0; j < Sh::NTW; j += 2) {
      if (j + 1 < Sh::NTW) {
        const int row = nbase + j * 8 + (m >> 1) * 8 + (lane & 7);
        const int col = ks * 16 + (m & 1) * 8;
        uint32_t bh0, bh1, bh2, bh3;
        ldsm_x4(smem_u32(wh) + wofs<R>(row, col), bh0, bh1, bh2, bh3);
        mma16816(acc[j], ah, bh0, bh1);
        mma16816(acc[j + 1], ah, bh2, bh3);
        if constexpr (LO) {
          uint32_t bl0, bl1, bl2, bl3;
          ldsm_x4(smem_u32(wl) + wofs<R>(row, col), bl0, bl1, bl2, bl3);
          mma16816(acc[j], ah, bl0, bl1);
          mma16816(acc[j + 1], ah, bl2, bl3);
        }
        mma16816(acc[j], al, bh0, bh1);
        mma16816(acc[j + 1], al, bh2, bh3);
      } else {   // a single n-tile left: b fragments read directly (two bf16 per 32-bit word)
        const int row = nbase + j * 8 + g;
        const int col = ks * 16 + 2 * t;
        const char* whb = reinterpret_cast<const char*>(wh);
        const char* wlb = reinterpret_cast<const char*>(wl);
        const uint32_t bh0 = *reinterpret_cast<const uint32_t*>(whb + wofs<R>(row, col));
        const uint32_t bh1 = *reinterpret_cast<const uint32_t*>(whb + wofs<R>(row, col + 8));
        mma16816(acc[j], ah, bh0, bh1);
        if constexpr (LO) {
          const uint32_t bl0 = *reinterpret_cast<const uint32_t*>(wlb + wofs<R>(row, col));
          const uint32_t bl1 = *reinterpret_cast<const uint32_t*>(wlb + wofs<R>(row, col + 8));
          mma16816(acc[j], ah, bl0, bl1);
        }
        mma16816(acc[j], al, bh0, bh1);
      }
    }
  }
}

// v = gelu(acc + bias) for this thread's outputs; written either as the next
// layer's hi / lo operand tiles or as fp32.  acc is cleared.
template <int R>
__device__ __forceinline__ void mlp_epilogue(float (*acc)[4], const float2* bias, __nv_bfloat16* oh,
                                             __nv_bfloat16* ol, float* of) {
  using Sh = RouterShape<R>;
  const int warp = warp_id(), lane = lane_id();
  if ((warp >> 1) >= Sh::NG) return;
  const int r0 = (warp & 1) * 16 + (lane >> 2);
  const int nbase = (warp >> 1) * (R / Sh::NG);
#pragma unroll
  for (int j = 0; j < Sh::NTW; ++j) {
    const int n = nbase + j * 8 + 2 * (lane & 3);
    float v[4];
    v[0] = gelu_exact(acc[j][0] + bias[j].x);
    v[1] = gelu_exact(acc[j][1] + bias[j].y);
    v[2] = gelu_exact(acc[j][2] + bias[j].x);
    v[3] = gelu_exact(acc[j][3] + bias[j].y);
    if (of) {
      *reinterpret_cast<float2*>(of + r0 * kZS + n) = make_float2(v[0], v[1]);
      *reinterpret_cast<float2*>(of + (r0 + 8) * kZS + n) = make_float2(v[2], v[3]);
    } else {
      float h[4], l[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) split_bf(v[i], h[i], l[i]);
      *reinterpret_cast<uint32_t*>(oh + r0 * kAS + n) = pack_bf2(h[0], h[1]);
      *reinterpret_cast<uint32_t*>(oh + (r0 + 8) * kAS + n) = pack_bf2(h[2], h[3]);
      *reinterpret_cast<uint32_t*>(ol + r0 * kAS + n) = pack_bf2(l[0], l[1]);
      *reinterpret_cast<uint32_t*>(ol + (r0 + 8) * kAS + n) = pack_bf2(l[2], l[3]);
    }
    acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  }
}

// Output classes padded to whole 8-wide MMA tiles.
__host__ __device__ constexpr int router_np(int e1) { return (e1 + 7) / 8 * 8; }

// fc1 / fc2 weights (fp32 [R][R]) -> bf16 hi and lo parts: wsplit = [layer][hi|lo][R][R];
// then out_proj (fp32 [E1][R]) -> [hi|lo][NP][R] with zero rows from E1 on;
// four elements per thread.  Block 0 also clears the router's per-class counts
// (a kernel, not a memset, keeps the launch chain programmatic).
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ fc1, const float* __restrict__ fc2,
                                                           const float* __restrict__ out_w, int e1,
                                                           __nv_bfloat16* __restrict__ wsplit, int R,
                                                           int* __restrict__ class_count, int* __restrict__ lo_any) {
  griddep_begin();
  if (blockIdx.x == 0 && threadIdx.x < e1) class_count[threadIdx.x] = 0;
  const int n4 = R * R / 4, r4 = R / 4, np = router_np(e1);
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  // lo_any[block]: whether any weight of this block's share has a nonzero lo
  // part (every block writes its word every launch)
  bool lo_nz = false;
  if (i < 2 * n4 + np * r4) {
  float4 x;
  __nv_bfloat16* hi;
  __nv_bfloat16* lo;
  int e4;
  if (i < 2 * n4) {
    const int layer = i / n4;
    e4 = i % n4;
    x = __ldg(reinterpret_cast<const float4*>(layer ? fc2 : fc1) + e4);
    hi = wsplit + (size_t)layer * 2 * R * R;
    lo = hi + R * R;
  } else {
    e4 = i - 2 * n4;
    const int row = e4 / r4;
    x = row < e1 ? __ldg(reinterpret_cast<const float4*>(out_w) + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
    hi = wsplit + (size_t)4 * R * R;
    lo = hi + (size_t)np * R;
  }
  const float hx = round_bf(x.x), hy = round_bf(x.y), hz = round_bf(x.z), hw = round_bf(x.w);
  reinterpret_cast<uint2*>(hi)[e4] = make_uint2(pack_bf2(hx, hy), pack_bf2(hz, hw));
  reinterpret_cast<uint2*>(lo)[e4] = make_uint2(pack_bf2(x.x - hx, x.y - hy), pack_bf2(x.z - hz, x.w - hw));
  lo_nz = (x.x != hx) || (x.y != hy) || (x.z != hz) || (x.w != hw);
  }
  lo_nz = __syncthreads_or(lo_nz);
  if (threadIdx.x == 0) lo_any[blockIdx.x] = lo_nz ? 1 : 0;
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1) router_kernel(const RouterParams p,
                                                             const __grid_constant__ CUtensorMap tmW) {
  using Sh = RouterShape<R>;
  constexpr int nch = R / Sh::KCH;
  griddep_begin();
  extern __shared__ __align__(16) float sm[];
  float* z = sm;                                                                // fp32 [kTM][kZS]
  __nv_bfloat16* zh = reinterpret_cast<__nv_bfloat16*>(z + kTM * kZS);          // bf16 hi [kTM][kAS]
  __nv_bfloat16* zl = zh + kTM * kAS;                                           // bf16 lo [kTM][kAS]
  // [2 stages][hi|lo][R][WS]; 1024-byte aligned for the swizzled TMA chunks
  __nv_bfloat16* wring = reinterpret_cast<__nv_bfloat16*>(
      Sh::TMA ? (reinterpret_cast<uintptr_t>(zl + kTM * kAS) + 1023) & ~uintptr_t(1023)
              : reinterpret_cast<uintptr_t>(zl + kTM * kAS));
  __shared__ uint64_t wfull[2];   // TMA mode: chunk landed in ring stage s
  const int E1 = p.E + 1;
  const int t0 = blockIdx.x * kTM;
  const int warp = warp_id(), lane = lane_id();
  const size_t n = (size_t)R * R;
  __shared__ int s_cnt[96], s_cls[kTM], s_rank[kTM];   // per-class counts of this CTA's tokens
  for (int c = threadIdx.x; c < 96; c += kThreads) s_cnt[c] = 0;
  // Weights that are bf16 values (a bf16 checkpoint) have zero lo parts: then
  // only the hi parts are loaded and the a.W_lo products are skipped (the
  // result is the same; the activations keep their hi / lo split).
  bool lo_w = false;
  if (warp == 0) {
    int any = 0;
    for (int i = lane; i < p.n_lo_words; i += 32) any |= p.lo_any[i];
    lo_w = __any_sync(0xffffffffu, any != 0);
  }
  lo_w = __syncthreads_or(lo_w);
  // weight chunk q of the fc1 -> fc2 sequence into ring stage q & 1: two TMA
  // boxes (hi, lo) of [R rows][64 columns] on the stage's barrier, issued by
  // thread 0; or (R = 32) one cp.async group of all threads
  auto stage_w = [&](int q) {
    if constexpr (Sh::TMA) {
      if (threadIdx.x == 0) {
        uint64_t* bar = &wfull[q & 1];
        mbar_arrive_expect_tx(bar, (lo_w ? 2 : 1) * Sh::CHUNK * (uint32_t)sizeof(__nv_bfloat16));
        const int row = (q / nch) * 2 * R;   // layer q / nch: hi rows, then lo rows
        tma_load_2d(wring + (q & 1) * 2 * Sh::CHUNK, &tmW, bar, (q % nch) * Sh::KCH, row);
        if (lo_w) tma_load_2d(wring + (q & 1) * 2 * Sh::CHUNK + Sh::CHUNK, &tmW, bar, (q % nch) * Sh::KCH, row + R);
      }
    } else {
      const __nv_bfloat16* whi = p.wsplit + (size_t)(q / nch) * 2 * n;
      stage_chunk<R>(wring + (q & 1) * 2 * Sh::CHUNK, whi, whi + n, (q % nch) * Sh::KCH);
    }
  };
  if constexpr (Sh::TMA) {
    if (threadIdx.x == 0) {
      mbar_init(&wfull[0], 1);
      mbar_init(&wfull[1], 1);
      fence_barrier_init();
      prefetch_tmap(&tmW);
    }
  }
  const WaitCtx wc = wait_ctx(p.status);
  stage_w(0);   // the first fc1 chunk streams in under the state assembly

  // router state r = down_proj partial sums (in slab order) + bias (+ previous
  // state * scale).  Each thread owns kPos float4 positions; the loads of two
  // slabs for all of them are issued before any add.  n_splits 0: the
  // down-projection's epilogue has written r itself (to r_out), read as is.
  {
    constexpr int R4 = R / 4;
    constexpr int kPos = (kTM * R4 + kThreads - 1) / kThreads;
    const size_t slab = (size_t)p.M * R4;
    const bool fused = p.n_splits == 0;
    const int ns = fused ? 1 : p.n_splits;
    const float4* part = reinterpret_cast<const float4*>(fused ? p.r_out : p.part);
    float4 v[kPos];
    size_t off[kPos];
    bool live[kPos], here[kPos];
#pragma unroll
    for (int u = 0; u < kPos; ++u) {
      const int i = threadIdx.x + u * kThreads;
      const int tt = i / R4, k4 = i % R4, t = t0 + tt;
      here[u] = i < kTM * R4;
      live[u] = here[u] && t < p.M;
      off[u] = (size_t)(live[u] ? t : 0) * R4 + k4;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int sp = 0; sp < ns; sp += 2) {
      float4 a0[kPos], a1[kPos];
#pragma unroll
      for (int u = 0; u < kPos; ++u) {
        a0[u] = part[sp * slab + off[u]];
        a1[u] = (sp + 1 < ns) ? part[(sp + 1) * slab + off[u]] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kPos; ++u) {
        v[u].x += a0[u].x; v[u].y += a0[u].y; v[u].z += a0[u].z; v[u].w += a0[u].w;
        v[u].x += a1[u].x; v[u].y += a1[u].y; v[u].z += a1[u].z; v[u].w += a1[u].w;
      }
    }
    float4 pv[kPos];
    if (p.prev && !fused) {
#pragma unroll
      for (int u = 0; u < kPos; ++u) pv[u] = reinterpret_cast<const float4*>(p.prev)[off[u]];
    }
#pragma unroll
    for (int u = 0; u < kPos; ++u) {
      const int i = threadIdx.x + u * kThreads;
      const int tt = i / R4, k4 = i % R4;
      if (!here[u]) continue;
      if (!fused) {
        const float4 bb = __ldg(reinterpret_cast<const float4*>(p.bias) + k4);
        v[u].x += bb.x; v[u].y += bb.y; v[u].z += bb.z; v[u].w += bb.w;
        if (p.prev) {
          const float4 sc = __ldg(reinterpret_cast<const float4*>(p.prev_scale) + k4);
          v[u].x = fmaf(pv[u].x, sc.x, v[u].x); v[u].y = fmaf(pv[u].y, sc.y, v[u].y);
          v[u].z = fmaf(pv[u].z, sc.z, v[u].z); v[u].w = fmaf(pv[u].w, sc.w, v[u].w);
        }
      }
      if (!live[u]) v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      else if (!fused) reinterpret_cast<float4*>(p.r_out)[off[u]] = v[u];
      *reinterpret_cast<float4*>(z + tt * kZS + k4 * 4) = v[u];
    }
  }
  // fc1 / fc2 bias pairs of this thread's outputs, loaded once
  float2 b1[Sh::NTW], b2[Sh::NTW];
  if ((warp >> 1) < Sh::NG) {
    const int nbase = (warp >> 1) * (R / Sh::NG) + 2 * (lane & 3);
#pragma unroll
    for (int j = 0; j < Sh::NTW; ++j) {
      b1[j] = make_float2(__ldg(p.fc1_b + nbase + j * 8), __ldg(p.fc1_b + nbase + j * 8 + 1));
      b2[j] = make_float2(__ldg(p.fc2_b + nbase + j * 8), __ldg(p.fc2_b + nbase + j * 8 + 1));
    }
  }
  __syncthreads();
  {  // router_mlp.norm (RMSNorm over R), one warp per token -> fc1's hi / lo operand
    float nw[R / 32];
#pragma unroll
    for (int j = 0; j < R / 32; ++j) nw[j] = __ldg(p.norm_w + lane + 32 * j);
    for (int tt = warp; tt < kTM; tt += kThreads / 32) {
      float zr[R / 32], ss = 0.f;
#pragma unroll
      for (int j = 0; j < R / 32; ++j) {
        zr[j] = z[tt * kZS + lane + 32 * j];
        ss += zr[j] * zr[j];
      }
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss / (float)R + p.eps);
#pragma unroll
      for (int j = 0; j < R / 32; ++j) {
        float h, l;
        split_bf(nw[j] * (zr[j] * inv), h, l);
        zh[tt * kAS + lane + 32 * j] = __float2bfloat16_rn(h);
        zl[tt * kAS + lane + 32 * j] = __float2bfloat16_rn(l);
      }
    }
  }
  // fc1 then fc2 (GELU after each): 2 * nch weight chunks through a two-stage
  // ring, chunk q + 1 in flight while chunk q is multiplied; the split out_proj
  // weight ([hi|lo][NP][R + 8], padded rows) follows the last chunk into the
  // stage that chunk leaves free (or its own region).
  const int NP = router_np(E1);
  constexpr int OWS = R + 8;
  const bool ow_in_ring = (size_t)2 * NP * OWS <= (size_t)2 * Sh::CHUNK;
  __nv_bfloat16* ow = ow_in_ring ? wring + ((2 * nch) & 1) * 2 * Sh::CHUNK : wring + 4 * Sh::CHUNK;
  float acc[Sh::NTW][4];
#pragma unroll
  for (int j = 0; j < Sh::NTW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  bool ok = true;   // TMA mode: false once a chunk wait has run out (status set)
  int n_staged = 1;  // TMA mode, thread 0: chunks whose copies were started
  for (int q = 0; q < 2 * nch; ++q) {
    if (q + 1 < 2 * nch) {
      // after a failed wait no further chunk is started (its stage may still
      // be receiving the chunk that never arrived in time)
      if (!Sh::TMA || ok) {
        stage_w(q + 1);
        ++n_staged;
      }
    } else {
      const __nv_bfloat16* ows = p.wsplit + (size_t)4 * R * R;   // [hi|lo][NP][R]
      for (int i = threadIdx.x; i < (lo_w ? 2 : 1) * NP * (R / 8); i += kThreads) {
        const int row = i / (R / 8), c = i % (R / 8);   // row over hi rows then lo rows
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(ow + row * OWS + c * 8)),
                     "l"(ows + (size_t)row * R + c * 8)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    if constexpr (Sh::TMA) {   // every thread sees chunk q land (bounded wait)
      if (ok && !mbar_wait(&wfull[q & 1], (uint32_t)(q >> 1) & 1u, wc)) ok = false;
    }
    __syncthreads();
    const __nv_bfloat16* wh = wring + (q & 1) * 2 * Sh::CHUNK;
    if (lo_w) mlp_chunk<R, true>(zh, zl, acc, wh, wh + Sh::CHUNK, q % nch);
    else mlp_chunk<R, false>(zh, zl, acc, wh, wh + Sh::CHUNK, q % nch);
    if (q == nch - 1) {   // fc1 done: its GELU output becomes fc2's operand (in place)
      __syncthreads();
      mlp_epilogue<R>(acc, b1, zh, zl, nullptr);
    } else if (q == 2 * nch - 1) {   // fc2 done: its GELU output becomes out_proj's operand
      __syncthreads();
      mlp_epilogue<R>(acc, b2, zh, zl, nullptr);
    }
    __syncthreads();
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if constexpr (Sh::TMA) {   // every chunk copy started has landed before the CTA can exit
    if (threadIdx.x == 0)
      for (int q = (n_staged > 2 ? n_staged - 2 : 0); q < n_staged; ++q)
        mbar_drain(&wfull[q & 1], (uint32_t)(q >> 1) & 1u, p.status);
  }
  __syncthreads();
  // out_proj (no bias) on tensor cores with the same hi / lo split: tile w < 2 * NP / 8
  // (warps stride over them) is rows 16 * (w & 1) .. + 16 by classes 8 * (w >> 1) .. + 8
  // over all of R; the logits go to shared memory (z, fp32 [kTM][kZS], free since
  // fc2's epilogue)
  for (int w = warp; w < 2 * (NP / 8); w += kThreads / 32) {
    const int mt = w & 1, nt = w >> 1;
    const int g = lane >> 2, tq = lane & 3;
    const int arow = mt * 16 + (lane & 15);
    const __nv_bfloat16* owh = ow + (nt * 8 + g) * OWS;
    const __nv_bfloat16* owl = owh + NP * OWS;
    float c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int ks = 0; ks < R / 16; ++ks) {
      const int acol = ks * 16 + (lane >> 4) * 8;
      uint32_t ah[4], al[4];
      ldsm_x4(smem_u32(zh + arow * kAS + acol), ah[0], ah[1], ah[2], ah[3]);
      ldsm_x4(smem_u32(zl + arow * kAS + acol), al[0], al[1], al[2], al[3]);
      const int col = ks * 16 + 2 * tq;
      const uint32_t bh0 = *reinterpret_cast<const uint32_t*>(owh + col);
      const uint32_t bh1 = *reinterpret_cast<const uint32_t*>(owh + col + 8);
      mma16816(c4, ah, bh0, bh1);
      if (lo_w) {
        const uint32_t bl0 = *reinterpret_cast<const uint32_t*>(owl + col);
        const uint32_t bl1 = *reinterpret_cast<const uint32_t*>(owl + col + 8);
        mma16816(c4, ah, bl0, bl1);
      }
      mma16816(c4, al, bh0, bh1);
    }
    const int r0 = mt * 16 + g, n0 = nt * 8 + 2 * tq;
    *reinterpret_cast<float2*>(z + r0 * kZS + n0) = make_float2(c4[0], c4[1]);
    *reinterpret_cast<float2*>(z + (r0 + 8) * kZS + n0) = make_float2(c4[2], c4[3]);
  }
  __syncthreads();
  // softmax and the choice, one warp per token
  for (int tt = warp; tt < kTM; tt += kThreads / 32) {
    const int t = t0 + tt;
    if (t >= p.M) continue;
    float l[3];
#pragma unroll
    for (int u = 0; u < 3; ++u) l[u] = (lane + 32 * u < E1) ? z[tt * kZS + lane + 32 * u] : -INFINITY;
    float mx = fmaxf(fmaxf(l[0], l[1]), l[2]);
    mx = warp_max(mx);
    float e[3], sum = 0.f;
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
        const float sc = pc + __ldg(p.balancing + c);
        if (sc > best) {
          best = sc;
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
      s_cls[tt] = cls;
      s_rank[tt] = atomicAdd(&s_cnt[cls], 1);   // place among this CTA's tokens of the class
    }
  }
  // one global add per class reserves this CTA's rows within the class
  __syncthreads();
  for (int c = threadIdx.x; c < E1; c += kThreads)
    if (s_cnt[c]) s_cnt[c] = atomicAdd(p.class_count + c, s_cnt[c]);
  __syncthreads();
  for (int tt = threadIdx.x; tt < kTM; tt += kThreads)
    if (t0 + tt < p.M) p.slot[t0 + tt] = s_cnt[s_cls[tt]] + s_rank[tt];
}

template <int R>
int launch_router_r(const RouterParams& p, cudaStream_t st) {
  using Sh = RouterShape<R>;
  const int np = router_np(p.E + 1);
  const int n_split = 2 * R * R / 4 + np * R / 4;
  if (p.n_lo_words != (n_split + 255) / 256) return ZAYA_ERR_UNSUPPORTED;
  launch_k(router_split_kernel, dim3((n_split + 255) / 256), dim3(256), 0, st, nullptr, 0, p.fc1_w, p.fc2_w, p.out_w,
           p.E + 1, p.wsplit, R, p.class_count, p.lo_any);
  const size_t ow_elems = (size_t)2 * np * (R + 8);
  const size_t smem = Sh::SMEM + (ow_elems <= (size_t)2 * Sh::CHUNK ? 0 : ow_elems * sizeof(__nv_bfloat16));
  if (smem > 227 * 1024) return ZAYA_ERR_UNSUPPORTED;
  CUtensorMap mw;   // wsplit as [4R rows (layer, hi|lo, row)][R columns], boxes of R rows x 64 columns
  memset(&mw, 0, sizeof(mw));
  if constexpr (Sh::TMA) {
    if (!p.status) return ZAYA_ERR_UNSUPPORTED;
    const int rc = make_tmap_bf16(&mw, p.wsplit, (uint64_t)4 * R, (uint64_t)R, (uint32_t)R);
    if (rc) return rc;
  }
  cudaFuncSetAttribute(router_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_k(router_kernel<R>, dim3((p.M + kTM - 1) / kTM), dim3(kThreads), smem, st, nullptr, 0, p, mw);
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

// One warp per token row: routed tokens copy their m_in row to the permuted
// row (all eight 16-byte loads of a lane in flight at once); skipped (and
// padding) tokens write merge 2 with a zero routed output.
__global__ void __launch_bounds__(256) dispatch_kernel(const DispatchParams p) {
  griddep_begin();
  if (status_peek(p.status)) return;   // a fault earlier in the block: no merge, cache_len not advanced
  const int t = blockIdx.x * 8 + warp_id();
  const int lane = lane_id();
  const int E1 = p.E + 1;
  // class offsets: exclusive prefix of the class counts (and, from CTA 0, the
  // expert offsets and tile prefix the expert GEMMs read)
  int cnt[3], tiles[3];
#pragma unroll
  for (int u = 0; u < 3; ++u) {
    const int c = lane + 32 * u;
    cnt[u] = c < E1 ? p.class_count[c] : 0;
    tiles[u] = c < p.E ? (cnt[u] + p.tile_rows - 1) / p.tile_rows : 0;
  }
  int off[3], toff[3], carry = 0, tcarry = 0;
#pragma unroll
  for (int u = 0; u < 3; ++u) {
    int inc = cnt[u], tinc = tiles[u];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, inc, o), b2 = __shfl_up_sync(0xffffffffu, tinc, o);
      if (lane >= o) {
        inc += a;
        tinc += b2;
      }
    }
    off[u] = carry + inc - cnt[u];
    toff[u] = tcarry + tinc - tiles[u];
    carry += __shfl_sync(0xffffffffu, inc, 31);
    tcarry += __shfl_sync(0xffffffffu, tinc, 31);
  }
  if (blockIdx.x == 0 && warp_id() == 0) {
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int c = lane + 32 * u;
      if (c < E1) {
        p.group_off[c] = off[u];
        p.mt_start[c] = toff[u];
      }
    }
    if (lane == 0) {
      p.group_off[E1] = carry;
      p.mt_start[E1] = tcarry;
    }
  }
  if (t >= p.M) return;
  const int H = p.H;
  const int per_row = H / 8;   // 16-byte chunks
  int c = p.cls[t];
  if (c < 0 || c > p.E) c = p.E;
  const int row = __shfl_sync(0xffffffffu, off[0], c & 31) * (c < 32) +
                  __shfl_sync(0xffffffffu, off[1], c & 31) * (c >= 32 && c < 64) +
                  __shfl_sync(0xffffffffu, off[2], c & 31) * (c >= 64) + p.slot[t];
  if (lane == 0) {
    p.pos[t] = row;
    p.perm[row] = t;
  }
  if (c < p.E && p.in_scale) {   // FP8 experts: the row as E4M3 codes of x / s_in
    const float s_in = __ldg(p.in_scale + 2 * c);
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.m_in) + (size_t)t * H);
    uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.x_perm) + (size_t)row * H);
    for (int ch = lane; ch < per_row; ch += 32) {
      const uint4 v = src[ch];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 a = unpack_bf2(w[2 * h]), b = unpack_bf2(w[2 * h + 1]);
        o[h] = (uint32_t)pack_e4m3x2(__fdiv_rn(a.x, s_in), __fdiv_rn(a.y, s_in)) |
               ((uint32_t)pack_e4m3x2(__fdiv_rn(b.x, s_in), __fdiv_rn(b.y, s_in)) << 16);
      }
      dst[ch] = make_uint2(o[0], o[1]);
    }
  } else if (c < p.E) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.m_in) + (size_t)t * H);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.x_perm) + (size_t)row * H);
    constexpr int kV = 8;
    for (int c0 = 0; c0 < per_row; c0 += 32 * kV) {
      uint4 v[kV];
#pragma unroll
      for (int k = 0; k < kV; ++k) {
        const int ch = c0 + k * 32 + lane;
        if (ch < per_row) v[k] = src[ch];
      }
#pragma unroll
      for (int k = 0; k < kV; ++k) {
        const int ch = c0 + k * 32 + lane;
        if (ch < per_row) dst[ch] = v[k];
      }
    }
  } else {
    // skip: no expert runs; mlp_output = bf16(hb * hs), out = mlp_output + (h + rb) * rs
    for (int ch = lane; ch < per_row; ch += 32) {
      float4* s4 = reinterpret_cast<float4*>(p.stream + (size_t)t * H + ch * 8);
      float cb[8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float4 x = s4[h];
        float* xp = &x.x;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = ch * 8 + 4 * h + j;
          const float contrib = round_bf(__ldg(p.merge_m + col) * __ldg(p.merge_m + H + col));
          cb[4 * h + j] = contrib;
          xp[j] = fmaf(xp[j] + __ldg(p.merge_m + 2 * H + col), __ldg(p.merge_m + 3 * H + col), contrib);
        }
        s4[h] = x;
      }
      if (p.tap_mlp_out) {
        uint4 u;
        u.x = pack_bf2(cb[0], cb[1]);
        u.y = pack_bf2(cb[2], cb[3]);
        u.z = pack_bf2(cb[4], cb[5]);
        u.w = pack_bf2(cb[6], cb[7]);
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.tap_mlp_out) + (size_t)t * H)[ch] = u;
      }
    }
  }
  if (p.cache_len_inc && lane == 0) p.cache_len_inc[t] += 1;
}

}  // namespace

int router_split_blocks(int R, int E) {
  const int n_split = 2 * R * R / 4 + router_np(E + 1) * R / 4;
  return (n_split + 255) / 256;
}

int launch_router(const RouterParams& p, cudaStream_t st) {
  if (p.M <= 0) return ZAYA_OK;
  if (p.E + 1 > 96 || p.n_splits < 0 || !p.wsplit || !p.class_count) return ZAYA_ERR_UNSUPPORTED;
  switch (p.R) {
    case 32: return launch_router_r<32>(p, st);
    case 64: return launch_router_r<64>(p, st);
    case 128: return launch_router_r<128>(p, st);
    case 256: return launch_router_r<256>(p, st);
    default: return ZAYA_ERR_UNSUPPORTED;
  }
}

int launch_dispatch(const DispatchParams& p, cudaStream_t st) {
  if (p.M <= 0) return ZAYA_OK;
  if (p.H % 8 || p.E + 1 > 96 || p.tile_rows <= 0) return ZAYA_ERR_UNSUPPORTED;
  launch_k(dispatch_kernel, dim3((unsigned)((p.M + 7) / 8)), dim3(256), 0, st, nullptr, 0, p);
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

}  // namespace zaya
