// CCA attention inputs: causal conv over q||k, the CCA mean residual,
// qk_norm with the key temperature, partial RoPE, the value heads with their
// delayed half, and the writes into the KV cache / conv_state / prev_hs.
//
// As the nnterp "zaya" page states it ("Queries and keys are convolved,
// normed to sqrt(head_dim) and the keys scaled"):
//   y[t,c]  = w[c,0] u[t-2,c] + w[c,1] u[t-1,c] + w[c,2] u[t,c] + b[c]   (u = q||k pre-conv)
//   q_h    += (u_q[h] + u_k[g(h)]) / 2;   k_g += mean over h served by g of that
//   q, k    -> x * sqrt(d) / max(|x|, eps);   k *= temp[g]
//   RoPE on dims [0, rot): pairs (i, i + rot/2), angle = fp32(pos * inv_freq[i])
//   v_g     = [v_current(t)[g*d/2 .. ] || v_delayed(t-1)[g*d/2 .. ]]
// conv_state [B,C,2] and prev_hs [B,H] carry the two previous tokens' pre-conv
// channels and the previous token's attention-norm output (ZAYA1-8B-JANGTQ2
// README, "Architecture Summary").
//
// Each lane owns d/32 consecutive dims of a head, so the head norm is a warp
// reduction and the RoPE pair exchange a shuffle.  Prefill: a CTA covers 16
// consecutive tokens with their pre-conv rows staged in shared memory.
// Decode: a CTA per sequence.  HBM-bound: ~3 KB read and ~3 KB written per
// token.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

template <int D>
struct Pre {
  // pre-conv value of channel c at token offset o (0: t, 1: t-1, 2: t-2)
  const __nv_bfloat16* qkv;
  size_t ld;
  const __nv_bfloat16* conv_state;  // decode history [C, 2]
  int tok, s, decode;
  const int* mask;
  bool real0, real1, real2;

  __device__ __forceinline__ float at(int c, int o) const {
    if (o == 0) return real0 ? bf2f(qkv[(size_t)tok * ld + c]) : 0.f;
    if (decode) return bf2f(conv_state[(size_t)c * 2 + (o == 2 ? 0 : 1)]);
    const bool r = (o == 1) ? real1 : real2;
    return r ? bf2f(qkv[(size_t)(tok - o) * ld + c]) : 0.f;
  }
};

// DPL consecutive bf16 (4- or 8-byte aligned) read as one load.
template <int DPL>
__device__ __forceinline__ void load_bf(const __nv_bfloat16* src, float (&y)[DPL]) {
  if constexpr (DPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    const float2 a = unpack_bf2(u.x), b = unpack_bf2(u.y);
    y[0] = a.x; y[1] = a.y; y[2] = b.x; y[3] = b.y;
  } else {
    const float2 a = unpack_bf2(*reinterpret_cast<const uint32_t*>(src));
    y[0] = a.x; y[1] = a.y;
  }
}
// N consecutive fp32 (16-byte aligned when N % 4 == 0) through the read-only path.
template <int N>
__device__ __forceinline__ void load_f(const float* __restrict__ src, float (&y)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src) + i);
      y[4 * i] = v.x; y[4 * i + 1] = v.y; y[4 * i + 2] = v.z; y[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const float2 v = __ldg(reinterpret_cast<const float2*>(src) + i);
      y[2 * i] = v.x; y[2 * i + 1] = v.y;
    }
  }
}

// DPL consecutive bf16 written as one 4- or 8-byte store.
template <int DPL>
__device__ __forceinline__ void store_bf(__nv_bfloat16* dst, const float (&y)[DPL]) {
  if constexpr (DPL == 4) {
    uint2 u;
    u.x = pack_bf2(y[0], y[1]);
    u.y = pack_bf2(y[2], y[3]);
    *reinterpret_cast<uint2*>(dst) = u;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf2(y[0], y[1]);
  }
}

template <int D>
__device__ __forceinline__ void rope_apply(float (&y)[D / 32], int lane, int pos, int rot, const float* inv_freq_tab) {
  constexpr int DPL = D / 32;
  if (rot <= 0) return;
  const int half = rot / 2;
  const int off = half / DPL;  // lane distance between the two dims of a pair
  const float posf = (float)pos;
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    const int j = lane * DPL + i;
    const bool lo = j < half;
    const bool in_rot = j < rot;
    int src = lo ? lane + off : lane - off;
    if (!in_rot) src = lane;
    const float partner = __shfl_sync(0xffffffffu, y[i], src);
    if (in_rot) {
      const int f = lo ? j : j - half;
      const float inv_freq = inv_freq_tab[f];
      const float ang = posf * inv_freq;
      float sn, cs;
      sincosf(ang, &sn, &cs);
      y[i] = lo ? (y[i] * cs - partner * sn) : (y[i] * cs + partner * sn);
    }
  }
}

// Decode (one token per sequence, history from conv_state) -- and the
// general per-token form: CTA = one token, one warp per head.
template <int D>
__global__ void __launch_bounds__(1024) cca_kernel(const CcaParams p) {
  constexpr int DPL = D / 32;
  griddep_begin();
  const int tok = blockIdx.x;
  const int b = p.decode ? tok : tok / p.S;
  const int s = p.decode ? 0 : tok % p.S;
  const int warp = warp_id(), lane = lane_id();
  const int nq = p.n_q, nkv = p.n_kv, rep = nq / nkv;
  const int C = (nq + nkv) * D;
  const auto* qkv = static_cast<const __nv_bfloat16*>(p.qkv);
  const size_t ld = (size_t)p.n_qkv;

  const int pos = p.decode ? p.cache_len[b] : s;
  // Decode appends at cache_len[b]: a position outside the cache is a fault
  // (a window ring takes any position >= 0, at slot pos % cache_cap).
  // Every CTA checks all sequences, so a call with one bad position writes no
  // sequence's cache, conv_state or prev_hs (the status word then makes the
  // rest of the block skip its work, and cache_len stays as it was).
  const bool ring = p.decode && p.ring;
  auto outside = [&](int c) { return c < 0 || (!ring && c >= p.cache_cap); };
  bool bad = false;
  if (p.decode) {
    for (int i = threadIdx.x; i < p.B; i += blockDim.x) bad |= outside(p.cache_len[i]);
  } else {
    bad = outside(pos);
  }
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0 && outside(pos)) set_status(p.status, ZAYA_ERR_DEVICE_RANGE);
    return;
  }
  const int slot = ring ? pos % p.cache_cap : pos;   // the cache row of this position
  Pre<D> pre;
  pre.qkv = qkv;
  pre.ld = ld;
  pre.conv_state = static_cast<const __nv_bfloat16*>(p.conv_state) + (size_t)b * C * 2;
  pre.tok = tok;
  pre.s = s;
  pre.decode = p.decode;
  pre.mask = p.mask;
  pre.real0 = p.decode || !p.mask || p.mask[tok] != 0;
  pre.real1 = !p.decode && s >= 1 && (!p.mask || p.mask[tok - 1] != 0);
  pre.real2 = !p.decode && s >= 2 && (!p.mask || p.mask[tok - 2] != 0);
  const bool last = p.decode || s == p.S - 1;
  auto* cstate = static_cast<__nv_bfloat16*>(p.conv_state) + (size_t)b * C * 2;
  const float sqrt_d = sqrtf((float)D);

  if (warp < nq + nkv) {
    // ------------------------------------------------ query head / key head
    const bool is_q = warp < nq;
    const int head = is_q ? warp : warp - nq;
    const int g = is_q ? warp / rep : head;
    float y[DPL];
    float u0[DPL], u1[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int j = lane * DPL + i;
      const int c = (is_q ? head * D : nq * D + head * D) + j;
      const float a0 = pre.at(c, 0), a1 = pre.at(c, 1), a2 = pre.at(c, 2);
      u0[i] = a0;
      u1[i] = a1;
      float acc;
      if (p.conv_y) {   // the two-stage conv, computed by the grouped-conv kernel
        acc = p.conv_y[(size_t)tok * C + c];
      } else {
        acc = __ldg(p.conv_b + c);
        acc = fmaf(__ldg(p.conv_w + 3 * c + 0), a2, acc);
        acc = fmaf(__ldg(p.conv_w + 3 * c + 1), a1, acc);
        acc = fmaf(__ldg(p.conv_w + 3 * c + 2), a0, acc);
      }
      if (p.cca_res) {
        const float kpre = pre.at(nq * D + g * D + j, 0);
        if (is_q) {
          acc += 0.5f * (a0 + kpre);
        } else {
          float qs = 0.f;
          for (int h = g * rep; h < (g + 1) * rep; ++h) qs += pre.at(h * D + j, 0);
          acc += 0.5f * (qs / (float)rep + kpre);
        }
      }
      y[i] = acc;
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) ss += y[i] * y[i];
    ss = warp_sum(ss);
    float scl = sqrt_d / fmaxf(sqrtf(ss), p.eps);
    if (!is_q) scl *= __ldg(p.k_temp + g);
#pragma unroll
    for (int i = 0; i < DPL; ++i) y[i] *= scl;
    rope_apply<D>(y, lane, pos, p.rot, p.inv_freq);

    __nv_bfloat16* dst;
    if (is_q) {
      const int Sq = p.decode ? 1 : p.S;
      const size_t off = (((size_t)b * nq + head) * Sq + (p.decode ? 0 : s)) * D + lane * DPL;
      dst = static_cast<__nv_bfloat16*>(p.q_out) + off;
      if (p.tap_q) {
        __nv_bfloat16* t = static_cast<__nv_bfloat16*>(p.tap_q) + off;
#pragma unroll
        for (int i = 0; i < DPL; ++i) t[i] = f2bf(y[i]);
      }
    } else if (p.decode && p.fp8) {   // the cache's E4M3 of the bf16 key
      dst = nullptr;
      uint8_t* d8 = static_cast<uint8_t*>(p.k_cache) + (((size_t)b * nkv + head) * p.cache_cap + slot) * D + lane * DPL;
#pragma unroll
      for (int i = 0; i < DPL; i += 2)
        *reinterpret_cast<uint16_t*>(d8 + i) = pack_e4m3x2(round_bf(y[i]), round_bf(y[i + 1]));
    } else {
      dst = static_cast<__nv_bfloat16*>(p.k_cache) + (((size_t)b * nkv + head) * p.cache_cap + slot) * D + lane * DPL;
    }
    if (dst) {
#pragma unroll
      for (int i = 0; i < DPL; ++i) dst[i] = f2bf(y[i]);
    }

    if (last) {  // conv_state <- pre-conv channels of tokens t-1, t
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const int c = (is_q ? head * D : nq * D + head * D) + lane * DPL + i;
        cstate[(size_t)c * 2 + 0] = f2bf(u1[i]);
        cstate[(size_t)c * 2 + 1] = f2bf(u0[i]);
      }
    }
  } else if (warp < nq + 2 * nkv) {
    // ------------------------------------------------ value head
    const int g = warp - nq - nkv;
    const int vc0 = nq * D + nkv * D;
    const int vd0 = vc0 + nkv * (D / 2);
    __nv_bfloat16* dst =
        static_cast<__nv_bfloat16*>(p.v_cache) + (((size_t)b * nkv + g) * p.cache_cap + slot) * D + lane * DPL;
    float vv[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int j = lane * DPL + i;
      float v;
      if (j < D / 2) {
        v = pre.real0 ? bf2f(qkv[(size_t)tok * ld + vc0 + g * (D / 2) + j]) : 0.f;
      } else {
        const int col = vd0 + g * (D / 2) + (j - D / 2);
        if (!p.v_delayed) {
          v = pre.real0 ? bf2f(qkv[(size_t)tok * ld + col]) : 0.f;
        } else if (p.decode) {
          v = bf2f(qkv[(size_t)(p.B + b) * ld + col]);  // projection of prev_hs
        } else {
          v = pre.real1 ? bf2f(qkv[(size_t)(tok - 1) * ld + col]) : 0.f;
        }
      }
      vv[i] = v;
    }
    if (p.decode && p.fp8) {   // the cache's E4M3 of the bf16 value
      uint8_t* d8 = static_cast<uint8_t*>(p.v_cache) + (((size_t)b * nkv + g) * p.cache_cap + slot) * D + lane * DPL;
#pragma unroll
      for (int i = 0; i < DPL; i += 2)
        *reinterpret_cast<uint16_t*>(d8 + i) = pack_e4m3x2(round_bf(vv[i]), round_bf(vv[i + 1]));
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) dst[i] = f2bf(vv[i]);
    }
    if (last && g == 0) {  // prev_hs <- attention_norm_output of this token
      const uint2* src = reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p.a_in) + (size_t)tok * p.H);
      uint2* ph = reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.prev_hs) + (size_t)b * p.H);
      for (int c = lane; c < p.H / 4; c += 32) ph[c] = src[c];
      if (!p.decode && lane == 0) p.cache_len[b] = p.S;
    }
  }
}


// Prefill: CTA = kTok consecutive tokens of one sequence.  The pre-conv rows
// t0-2 .. t0+kTok-1 (all q/k/v projection columns, padding rows zeroed) are
// staged once in shared memory, so every conv tap, the CCA residual and the
// delayed value half read shared memory; RoPE cos/sin are tabled once per
// (token, frequency) and shared by all heads.
constexpr int kTok = 16;

template <int D>
__global__ void __launch_bounds__(512) cca_prefill_kernel(const CcaParams p) {
  constexpr int DPL = D / 32;
  griddep_begin();
  if (p.zero_words && blockIdx.x == 0 && blockIdx.y == 0)   // the attention's merge counters
    for (int i = threadIdx.x; i < p.n_zero_words; i += blockDim.x) p.zero_words[i] = 0;
  extern __shared__ __align__(16) uint8_t sm[];
  const int nq = p.n_q, nkv = p.n_kv, rep = nq / nkv;
  const int C = (nq + nkv) * D;
  const int ld = p.n_qkv;
  const int b = blockIdx.y;
  const int s0 = blockIdx.x * kTok;
  const int half = p.rot / 2;
  auto* u = reinterpret_cast<__nv_bfloat16*>(sm);                              // [kTok + 2][ld]
  float* inv_f = reinterpret_cast<float*>(sm + (size_t)(kTok + 2) * ld * 2);   // [half]
  float2* cs = reinterpret_cast<float2*>(inv_f + 64);                          // [kTok][half]
  const auto* qkv = static_cast<const __nv_bfloat16*>(p.qkv);
  const size_t row0 = (size_t)b * p.S;

  // stage rows s0-2 .. s0+kTok-1 with cp.async (16-byte vectors, all issued before
  // one wait; zero-filled outside the sequence and at padding)
  const int vec_per_row = ld / 8;
  for (int i = threadIdx.x; i < (kTok + 2) * vec_per_row; i += blockDim.x) {
    const int r = i / vec_per_row, c = i % vec_per_row;
    const int s = s0 - 2 + r;
    const bool valid = s >= 0 && s < p.S && (!p.mask || p.mask[row0 + s] != 0);
    const __nv_bfloat16* src = qkv + (row0 + (valid ? s : 0)) * ld + c * 8;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(u + (size_t)r * ld + c * 8)),
                 "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int f = threadIdx.x; f < half; f += blockDim.x) inv_f[f] = p.inv_freq[f];
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  for (int i = threadIdx.x; i < kTok * half; i += blockDim.x) {
    const int tt = i / half, f = i % half;
    float sn, c;
    sincosf((float)(s0 + tt) * inv_f[f], &sn, &c);
    cs[i] = make_float2(c, sn);
  }
  __syncthreads();

  const int warp = warp_id(), lane = lane_id();
  const int n_heads = nq + 2 * nkv;
  const float sqrt_d = sqrtf((float)D);
  for (int task = warp; task < kTok * n_heads; task += blockDim.x / 32) {
    const int tt = task / n_heads, head = task % n_heads;
    const int s = s0 + tt;
    if (s >= p.S) continue;
    const __nv_bfloat16* ut = u + (size_t)(tt + 2) * ld;   // token t
    const __nv_bfloat16* u1 = ut - ld;                      // t - 1
    const __nv_bfloat16* u2 = ut - 2 * ld;                  // t - 2
    if (head < nq + nkv) {
      const bool is_q = head < nq;
      const int hh = is_q ? head : head - nq;
      const int g = is_q ? head / rep : hh;
      const int cbase = (is_q ? hh * D : nq * D + hh * D) + lane * DPL;
      float y[DPL], a0[DPL], a1[DPL], a2[DPL], w[3 * DPL], bias[DPL];
      load_bf<DPL>(ut + cbase, a0);
      load_bf<DPL>(u1 + cbase, a1);
      load_bf<DPL>(u2 + cbase, a2);
      if (p.conv_y) {   // the two-stage conv, computed by the grouped-conv kernel
        load_f<DPL>(p.conv_y + (row0 + s) * C + cbase, y);
      } else {
        load_f<3 * DPL>(p.conv_w + 3 * cbase, w);
        load_f<DPL>(p.conv_b + cbase, bias);
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
          float acc = bias[i];
          acc = fmaf(w[3 * i + 0], a2[i], acc);
          acc = fmaf(w[3 * i + 1], a1[i], acc);
          acc = fmaf(w[3 * i + 2], a0[i], acc);
          y[i] = acc;
        }
      }
      if (p.cca_res) {
        float kpre[DPL];
        load_bf<DPL>(ut + nq * D + g * D + lane * DPL, kpre);
        if (is_q) {
#pragma unroll
          for (int i = 0; i < DPL; ++i) y[i] += 0.5f * (a0[i] + kpre[i]);
        } else {
          float qs[DPL];
#pragma unroll
          for (int i = 0; i < DPL; ++i) qs[i] = 0.f;
          for (int h2 = g * rep; h2 < (g + 1) * rep; ++h2) {
            float qh[DPL];
            load_bf<DPL>(ut + h2 * D + lane * DPL, qh);
#pragma unroll
            for (int i = 0; i < DPL; ++i) qs[i] += qh[i];
          }
#pragma unroll
          for (int i = 0; i < DPL; ++i) y[i] += 0.5f * (qs[i] / (float)rep + kpre[i]);
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) ss += y[i] * y[i];
      ss = warp_sum(ss);
      float scl = sqrt_d / fmaxf(sqrtf(ss), p.eps);
      if (!is_q) scl *= __ldg(p.k_temp + g);
#pragma unroll
      for (int i = 0; i < DPL; ++i) y[i] *= scl;
      if (half > 0) {   // rotate-half over dims [0, rot)
        const int off = half / DPL;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
          const int j = lane * DPL + i;
          const bool lo = j < half, in_rot = j < p.rot;
          const int src = in_rot ? (lo ? lane + off : lane - off) : lane;
          const float partner = __shfl_sync(0xffffffffu, y[i], src);
          if (in_rot) {
            const float2 e = cs[tt * half + (lo ? j : j - half)];
            y[i] = lo ? (y[i] * e.x - partner * e.y) : (y[i] * e.x + partner * e.y);
          }
        }
      }
      __nv_bfloat16* dst;
      if (is_q) {
        const size_t off = (((size_t)b * nq + hh) * p.S + s) * D + lane * DPL;
        dst = static_cast<__nv_bfloat16*>(p.q_out) + off;
        if (p.tap_q) store_bf<DPL>(static_cast<__nv_bfloat16*>(p.tap_q) + off, y);
      } else {
        dst = static_cast<__nv_bfloat16*>(p.k_cache) + (((size_t)b * nkv + hh) * p.cache_cap + s) * D + lane * DPL;
      }
      store_bf<DPL>(dst, y);
      if (s == p.S - 1) {   // conv_state <- pre-conv channels of tokens S-2, S-1
        auto* cst = static_cast<__nv_bfloat16*>(p.conv_state) + (size_t)b * C * 2;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
          cst[(size_t)(cbase + i) * 2 + 0] = f2bf(a1[i]);
          cst[(size_t)(cbase + i) * 2 + 1] = f2bf(a0[i]);
        }
      }
    } else {
      const int g = head - nq - nkv;
      const int vc0 = nq * D + nkv * D;
      const int vd0 = vc0 + nkv * (D / 2);
      __nv_bfloat16* dst =
          static_cast<__nv_bfloat16*>(p.v_cache) + (((size_t)b * nkv + g) * p.cache_cap + s) * D + lane * DPL;
      float vv[DPL];
      const int j0 = lane * DPL;   // DPL consecutive dims lie in one half of the head
      if (j0 < D / 2)
        load_bf<DPL>(ut + vc0 + g * (D / 2) + j0, vv);
      else
        load_bf<DPL>((p.v_delayed ? u1 : ut) + vd0 + g * (D / 2) + (j0 - D / 2), vv);
      store_bf<DPL>(dst, vv);
      if (s == p.S - 1 && g == 0) {   // prev_hs <- attention_norm_output of token S-1
        const uint2* src = reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p.a_in) + (row0 + s) * p.H);
        uint2* ph = reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.prev_hs) + (size_t)b * p.H);
        for (int c = lane; c < p.H / 4; c += 32) ph[c] = src[c];
        if (lane == 0) p.cache_len[b] = p.S;
      }
    }
  }
}

// Prefill, streaming form: a thread owns 8 consecutive channels of one q/k
// head (the d/8 threads of a head are adjacent lanes, so the head norm and the
// RoPE pair exchange are shuffles inside that lane group) and walks kPerGroup
// consecutive tokens, reading each token's three conv inputs (t-2, t-1, t)
// and its taps and bias from shared memory (no values carried in registers:
// 768 threads leave 85 registers a thread); kGroups such thread groups split
// the CTA's kStream staged tokens.  Value heads: d/8 threads per
// kv head copy the current / delayed halves.  Needs rot % 16 == 0 (a thread's
// 8 dims are all inside or all outside the rotated range).
constexpr int kGroups = 4;
constexpr int kPerGroup = 7;
constexpr int kStream = kGroups * kPerGroup;   // 28 tokens: S = 4096 fills the 148 SMs in one round

__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&y)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(src);
  const float2 a = unpack_bf2(v.x), b = unpack_bf2(v.y), c = unpack_bf2(v.z), d = unpack_bf2(v.w);
  y[0] = a.x; y[1] = a.y; y[2] = b.x; y[3] = b.y; y[4] = c.x; y[5] = c.y; y[6] = d.x; y[7] = d.y;
}
__device__ __forceinline__ uint4 pack8(const float (&y)[8]) {
  return make_uint4(pack_bf2(y[0], y[1]), pack_bf2(y[2], y[3]), pack_bf2(y[4], y[5]), pack_bf2(y[6], y[7]));
}

template <int D>
__global__ void __launch_bounds__(768, 1) cca_stream_kernel(const __grid_constant__ CcaParams p) {
  constexpr int LPH = D / 8;   // threads per head
  griddep_begin();
  if (p.zero_words && blockIdx.x == 0 && blockIdx.y == 0)   // the attention's merge counters
    for (int i = threadIdx.x; i < p.n_zero_words; i += blockDim.x) p.zero_words[i] = 0;
  extern __shared__ __align__(16) uint8_t sm[];
  const int nq = p.n_q, nkv = p.n_kv, rep = nq / nkv;
  const int C = (nq + nkv) * D;
  const int ld = p.n_qkv;
  const int b = blockIdx.y;
  const int s0 = blockIdx.x * kStream;
  const int half = p.rot / 2;
  auto* u = reinterpret_cast<__nv_bfloat16*>(sm);                                 // [kStream + 2][ld]
  float2* cs = reinterpret_cast<float2*>(sm + (size_t)(kStream + 2) * ld * 2);    // [kStream][half]
  float* cbias = reinterpret_cast<float*>(cs + kStream * half);                    // [C]
  float* cw = cbias + C;                                                           // [C][3] conv taps
  const auto* qkv = static_cast<const __nv_bfloat16*>(p.qkv);
  const size_t row0 = (size_t)b * p.S;

  // rows s0-2 .. s0+kStream-1 (zero outside the sequence and at padding), one
  // cp.async wait; (row, 16-byte column) advance by blockDim.x vectors a step
  const int vec_per_row = ld / 8;
  const int dr = blockDim.x / vec_per_row, dc = blockDim.x % vec_per_row;
  for (int r = threadIdx.x / vec_per_row, c = threadIdx.x % vec_per_row; r < kStream + 2; r += dr, c += dc) {
    if (c >= vec_per_row) {
      c -= vec_per_row;
      ++r;
      if (r >= kStream + 2) break;
    }
    const int s = s0 - 2 + r;
    const bool valid = s >= 0 && s < p.S && (!p.mask || p.mask[row0 + s] != 0);
    const __nv_bfloat16* src = qkv + (row0 + (valid ? s : 0)) * ld + c * 8;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(u + (size_t)r * ld + c * 8)),
                 "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int i = threadIdx.x; i < kStream * half; i += blockDim.x) {
    const int tt = i / half, f = i % half;
    float sn, c;
    sincosf((float)(s0 + tt) * p.inv_freq[f], &sn, &c);
    cs[i] = make_float2(c, sn);
  }
  const int gthreads = blockDim.x / kGroups;              // a multiple of 32
  const int grp = threadIdx.x / gthreads, tid = threadIdx.x % gthreads, lane = lane_id();
  const int tt0 = grp * kPerGroup;                        // this group's first token
  const int n_qk = (nq + nkv) * LPH;
  // conv bias and taps of the q||k channels into shared memory (read by every
  // group each token, which keeps the token loop's registers below the cap
  // of 768 threads per SM), loaded under the staging
  const int head = tid / LPH, l = tid % LPH;
  const int cb = head * D + l * 8;
  if (!p.conv_y) {
    for (int i = threadIdx.x; i < C / 4; i += blockDim.x)
      reinterpret_cast<float4*>(cbias)[i] = __ldg(reinterpret_cast<const float4*>(p.conv_b) + i);
    for (int i = threadIdx.x; i < 3 * C / 4; i += blockDim.x)
      reinterpret_cast<float4*>(cw)[i] = __ldg(reinterpret_cast<const float4*>(p.conv_w) + i);
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  if (tid < n_qk) {
    const bool is_q = head < nq;
    const int hh = is_q ? head : head - nq;
    const int g = is_q ? head / rep : hh;
    const unsigned gmask = ((1u << LPH) - 1u) << (lane & ~(LPH - 1));   // this head's lanes
    const float scl0 = sqrtf((float)D) * (is_q ? 1.f : __ldg(p.k_temp + g));
    const float inv_rep = 1.0f / (float)rep;
    const float eps2 = p.eps * p.eps, inv_eps = 1.0f / p.eps;
    const int j0 = l * 8;
    const bool in_rot = j0 < p.rot, lo = j0 < half;
    const int src_lane = in_rot ? (lo ? lane + half / 8 : lane - half / 8) : lane;
    const int f0 = lo ? j0 : j0 - half;
    const int kcb = nq * D + g * D + l * 8;   // the group's key channels (query residual)
    const float4* wq = reinterpret_cast<const float4*>(cw + 3 * cb);   // taps (t-2, t-1, t) per channel
    __nv_bfloat16* dst = is_q ? static_cast<__nv_bfloat16*>(p.q_out) + (((size_t)b * nq + hh) * p.S + s0) * D + j0
                              : static_cast<__nv_bfloat16*>(p.k_cache) + (((size_t)b * nkv + hh) * p.cache_cap + s0) * D + j0;
    __nv_bfloat16* tap = (is_q && p.tap_q)
                             ? static_cast<__nv_bfloat16*>(p.tap_q) + (((size_t)b * nq + hh) * p.S + s0) * D + j0
                             : nullptr;
#pragma unroll 1
    for (int k = 0; k < kPerGroup; ++k) {
      const int tt = tt0 + k;
      const int s = s0 + tt;
      if (s >= p.S) break;   // uniform over the head's lanes
      const __nv_bfloat16* row = u + (size_t)(tt + 2) * ld;
      float x1[8], x0[8], y[8];
      load8(row - ld + cb, x1);
      load8(row + cb, x0);
      if (p.conv_y) {   // the two-stage conv, computed by the grouped-conv kernel
        const float4* cy = reinterpret_cast<const float4*>(p.conv_y + (row0 + s) * C + cb);
        const float4 y0 = cy[0], y1 = cy[1];
        y[0] = y0.x; y[1] = y0.y; y[2] = y0.z; y[3] = y0.w; y[4] = y1.x; y[5] = y1.y; y[6] = y1.z; y[7] = y1.w;
      } else {
        float x2[8], wv[24];
        load8(row - 2 * ld + cb, x2);
#pragma unroll
        for (int i = 0; i < 6; ++i) {
          const float4 v = wq[i];
          wv[4 * i] = v.x; wv[4 * i + 1] = v.y; wv[4 * i + 2] = v.z; wv[4 * i + 3] = v.w;
        }
        const float4 bb0 = reinterpret_cast<const float4*>(cbias + cb)[0];
        const float4 bb1 = reinterpret_cast<const float4*>(cbias + cb)[1];
        const float bb[8] = {bb0.x, bb0.y, bb0.z, bb0.w, bb1.x, bb1.y, bb1.z, bb1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float acc = bb[i];
          acc = fmaf(wv[3 * i], x2[i], acc);
          acc = fmaf(wv[3 * i + 1], x1[i], acc);
          acc = fmaf(wv[3 * i + 2], x0[i], acc);
          y[i] = acc;
        }
      }
      if (p.cca_res) {
        if (is_q) {
          float kp[8];
          load8(row + kcb, kp);
#pragma unroll
          for (int i = 0; i < 8; ++i) y[i] += 0.5f * (x0[i] + kp[i]);
        } else {
          float qs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          for (int h2 = g * rep; h2 < (g + 1) * rep; ++h2) {
            float qh[8];
            load8(row + h2 * D + l * 8, qh);
#pragma unroll
            for (int i = 0; i < 8; ++i) qs[i] += qh[i];
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) y[i] += 0.5f * (qs[i] * inv_rep + x0[i]);
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(y[i], y[i], ss);
#pragma unroll
      for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(gmask, ss, o);
      const float scl = scl0 * (ss > eps2 ? rsqrtf(ss) : inv_eps);   // sqrt(d) / max(|y|, eps)
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] *= scl;
      if (half > 0) {   // rotate-half over dims [0, rot)
        // pair by pair: both lanes of a pair read each other's value before either writes
        const float4* e4 = reinterpret_cast<const float4*>(cs + tt * half + (in_rot ? f0 : 0));
        const float sgn = lo ? -1.f : 1.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float pa = __shfl_sync(gmask, y[2 * i], src_lane);
          const float pb = __shfl_sync(gmask, y[2 * i + 1], src_lane);
          if (in_rot) {
            const float4 e = e4[i];   // (cos, sin) of dims 2i and 2i + 1
            y[2 * i] = fmaf(sgn * pa, e.y, y[2 * i] * e.x);
            y[2 * i + 1] = fmaf(sgn * pb, e.w, y[2 * i + 1] * e.z);
          }
        }
      }
      const uint4 o = pack8(y);
      *reinterpret_cast<uint4*>(dst + (size_t)tt * D) = o;
      if (tap) *reinterpret_cast<uint4*>(tap + (size_t)tt * D) = o;
      if (s == p.S - 1) {   // conv_state <- pre-conv channels of tokens S-2, S-1
        auto* cst = static_cast<__nv_bfloat16*>(p.conv_state) + (size_t)b * C * 2 + (size_t)cb * 2;
        uint4 c0, c1;
        c0.x = pack_bf2(x1[0], x0[0]); c0.y = pack_bf2(x1[1], x0[1]);
        c0.z = pack_bf2(x1[2], x0[2]); c0.w = pack_bf2(x1[3], x0[3]);
        c1.x = pack_bf2(x1[4], x0[4]); c1.y = pack_bf2(x1[5], x0[5]);
        c1.z = pack_bf2(x1[6], x0[6]); c1.w = pack_bf2(x1[7], x0[7]);
        reinterpret_cast<uint4*>(cst)[0] = c0;
        reinterpret_cast<uint4*>(cst)[1] = c1;
      }
    }
  } else if (tid < n_qk + nkv * LPH) {
    const int vt = tid - n_qk, g = vt / LPH, j0 = (vt % LPH) * 8;
    const int vc0 = nq * D + nkv * D;          // current halves
    const int vd0 = vc0 + nkv * (D / 2);       // delayed halves (from token t-1)
    auto* dst = static_cast<__nv_bfloat16*>(p.v_cache) + (((size_t)b * nkv + g) * p.cache_cap + s0) * D + j0;
    for (int tt = tt0; tt < tt0 + kPerGroup; ++tt) {
      const int s = s0 + tt;
      if (s >= p.S) break;
      const __nv_bfloat16* row = u + (size_t)(tt + 2) * ld;
      const __nv_bfloat16* src = (j0 < D / 2) ? row + vc0 + g * (D / 2) + j0
                                              : (p.v_delayed ? row - ld : row) + vd0 + g * (D / 2) + (j0 - D / 2);
      *reinterpret_cast<uint4*>(dst + (size_t)tt * D) = *reinterpret_cast<const uint4*>(src);
      if (s == p.S - 1 && g == 0) {   // prev_hs <- attention_norm_output of token S-1
        const uint4* hs = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.a_in) + (row0 + s) * p.H);
        uint4* ph = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.prev_hs) + (size_t)b * p.H);
        for (int c = vt; c < p.H / 8; c += LPH) ph[c] = hs[c];
        if (vt == 0) p.cache_len[b] = p.S;
      }
    }
  }
}

}  // namespace

int launch_cca(const CcaParams& p, cudaStream_t st) {
  const int tokens = p.decode ? p.B : p.B * p.S;
  if (tokens <= 0) return ZAYA_OK;
  const int threads = 32 * (p.n_q + 2 * p.n_kv);
  if (threads > 1024 || p.rot / 2 > 64 || p.n_qkv % 8) return ZAYA_ERR_UNSUPPORTED;
  if (!p.decode && (p.d == 128 || p.d == 64) && p.rot % 16 == 0 && p.H % 8 == 0) {
    const int lph = p.d / 8;
    const int nthr = kGroups * (((p.n_q + 2 * p.n_kv) * lph + 31) / 32 * 32);
    const size_t smem = (size_t)(kStream + 2) * p.n_qkv * 2 + (size_t)kStream * (p.rot / 2) * 8 +
                        (size_t)(p.n_q + p.n_kv) * p.d * 4 * 4;   // bias + three taps per q||k channel
    if (nthr <= 768 && smem <= 227 * 1024) {
      const dim3 grid((p.S + kStream - 1) / kStream, p.B);
      if (p.d == 128) {
        cudaFuncSetAttribute(cca_stream_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_k(cca_stream_kernel<128>, grid, dim3(nthr), smem, st, nullptr, 0, p);
      } else {
        cudaFuncSetAttribute(cca_stream_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_k(cca_stream_kernel<64>, grid, dim3(nthr), smem, st, nullptr, 0, p);
      }
      return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
    }
  }
  if (!p.decode) {
    const size_t smem = (size_t)(kTok + 2) * p.n_qkv * 2 + 64 * 4 + (size_t)kTok * (p.rot / 2) * 8;
    const dim3 grid((p.S + kTok - 1) / kTok, p.B);
    if (p.d == 128) {
      cudaFuncSetAttribute(cca_prefill_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      launch_k(cca_prefill_kernel<128>, grid, dim3(512), smem, st, nullptr, 0, p);
    } else if (p.d == 64) {
      cudaFuncSetAttribute(cca_prefill_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      launch_k(cca_prefill_kernel<64>, grid, dim3(512), smem, st, nullptr, 0, p);
    } else {
      return ZAYA_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
  }
  if (p.d == 128)
    launch_k(cca_kernel<128>, dim3(tokens), dim3(threads), 0, st, nullptr, 0, p);
  else if (p.d == 64)
    launch_k(cca_kernel<64>, dim3(tokens), dim3(threads), 0, st, nullptr, 0, p);
  else
    return ZAYA_ERR_UNSUPPORTED;
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}


namespace {

// One thread per 8 values (16 bytes of bf16) of a kept row: K and V of
// positions max(0, S - cap) .. S-1 of every (sequence, kv head), to slot p
// (ring: p % cap), as bf16 or as E4M3 bytes of the bf16 values.
__global__ void __launch_bounds__(256) cache_store_kernel(const uint4* __restrict__ k_lin,
                                                          const uint4* __restrict__ v_lin, void* __restrict__ k_cache,
                                                          void* __restrict__ v_cache, int BG, int S, int cap, int vpr,
                                                          int ring, int fp8, int* status) {
  griddep_begin();
  if (status_peek(status)) return;
  const int keep = S < cap ? S : cap;
  const long total = (long)BG * keep * vpr;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const int v = (int)(i % vpr);
    const long r = i / vpr;
    const int bg = (int)(r / keep);
    const int pos = S - keep + (int)(r % keep);
    const size_t src = ((size_t)bg * S + pos) * vpr + v;
    const size_t dst = ((size_t)bg * cap + (ring ? pos % cap : pos)) * vpr + v;
    const uint4 kx = k_lin[src], vx = v_lin[src];
    if (fp8) {
      auto enc = [](const uint4& x) {
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t o[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 a = unpack_bf2(w[2 * h]), c = unpack_bf2(w[2 * h + 1]);
          o[h] = (uint32_t)pack_e4m3x2(a.x, a.y) | ((uint32_t)pack_e4m3x2(c.x, c.y) << 16);
        }
        return make_uint2(o[0], o[1]);
      };
      static_cast<uint2*>(k_cache)[dst] = enc(kx);
      static_cast<uint2*>(v_cache)[dst] = enc(vx);
    } else {
      static_cast<uint4*>(k_cache)[dst] = kx;
      static_cast<uint4*>(v_cache)[dst] = vx;
    }
  }
}

}  // namespace

int launch_cache_store(const void* k_lin, const void* v_lin, void* k_cache, void* v_cache, int B, int n_kv, int S,
                       int cap, int d, int ring, int fp8, int* status, cudaStream_t st) {
  if (B <= 0 || S <= 0) return ZAYA_OK;
  if (cap <= 0 || d % 8) return ZAYA_ERR_UNSUPPORTED;
  const int vpr = d / 8;
  const long total = (long)B * n_kv * (S < cap ? S : cap) * vpr;
  const int blocks = (int)((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  launch_k(cache_store_kernel, dim3(blocks), dim3(256), 0, st, nullptr, 0, static_cast<const uint4*>(k_lin),
           static_cast<const uint4*>(v_lin), k_cache, v_cache, B * n_kv, S, cap, vpr, ring, fp8, status);
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

}  // namespace zaya
