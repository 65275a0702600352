// RMSNorm of the fp32 stream and the embedding gather.
//
// A block norm casts the fp32 stream to its weight's dtype (bf16) and norms
// it (nnterp "zaya" page, "The stream is float32 whatever the load"):
//   out = bf16(w * xb / sqrt(mean(xb^2) + eps)),  xb = bf16(x).
// H a multiple of 512: one 128-thread CTA per row, the row in registers
// (rmsnorm_row_kernel).  Other widths: one warp per row, float4 loads in
// groups; the row is read twice (sum of squares, then the output) so that no
// thread keeps it in registers and four 8-warp CTAs fit an SM; the second
// read is served from cache; the weight is staged in shared memory.
// HBM-bound (4 bytes read + 2 bytes written per element).
// The norms are launched in plain stream order, not as programmatic
// dependents: with their small CTAs waiting beside a CTA-pair GEMM (the
// previous block's expert down projection) and the next CTA-pair GEMM (the
// q/k/v projection) waiting on them in turn, a 40-block prefill stack at
// S = 32768 stopped making progress in about one stack in three; launched in
// stream order, 30 stacks of 30 completed (as they also did with the pair
// GEMMs launched in stream order instead).
#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

template <int CHUNKS>  // H = CHUNKS * 128
__global__ void __launch_bounds__(256, 4) rmsnorm_kernel(const float* __restrict__ x, int row_mul, int row_add,
                                                         const __nv_bfloat16* __restrict__ w,
                                                         __nv_bfloat16* __restrict__ out,
                                                         __nv_bfloat16* __restrict__ tap, int M, float eps,
                                                         const __nv_bfloat16* __restrict__ copy_src, int n_copy) {
  constexpr int H = CHUNKS * 128;
  constexpr int G = CHUNKS < 8 ? CHUNKS : 8;   // float4 loads in flight per group
  __shared__ __align__(16) __nv_bfloat16 ws[H];   // the norm weight, staged once per CTA
  griddep_begin();
  const int row = blockIdx.x * 8 + warp_id();
  const int lane = lane_id();
  for (int i = threadIdx.x; i < H / 8; i += blockDim.x)
    reinterpret_cast<uint4*>(ws)[i] = __ldg(reinterpret_cast<const uint4*>(w) + i);
  __syncthreads();
  if (row >= M + n_copy) return;
  if (row >= M) {  // verbatim copy rows (decode: prev_hs feeds the delayed values)
    const uint2* src = reinterpret_cast<const uint2*>(copy_src + (size_t)(row - M) * H);
    uint2* dst = reinterpret_cast<uint2*>(out + (size_t)row * H);
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) dst[c * 32 + lane] = src[c * 32 + lane];
    return;
  }
  const int src_row = row * row_mul + row_add;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)src_row * H);
  // pass 1: sum of squares of bf16(x); pass 2 reads the row again (now in L2 /
  // L1), so no thread holds the row in registers
  float ss = 0.f;
#pragma unroll 1
  for (int c0 = 0; c0 < CHUNKS; c0 += G) {
    float4 t[G];
#pragma unroll
    for (int c = 0; c < G; ++c) t[c] = xr[(c0 + c) * 32 + lane];
#pragma unroll
    for (int c = 0; c < G; ++c) {
      const float a0 = round_bf(t[c].x), a1 = round_bf(t[c].y), a2 = round_bf(t[c].z), a3 = round_bf(t[c].w);
      ss += a0 * a0 + a1 * a1 + a2 * a2 + a3 * a3;
    }
  }
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss / (float)H + eps);
  const uint2* wr = reinterpret_cast<const uint2*>(ws);
  uint2* orow = reinterpret_cast<uint2*>(out + (size_t)row * H);
  uint2* trow = tap ? reinterpret_cast<uint2*>(tap + (size_t)row * H) : nullptr;
#pragma unroll 1
  for (int c0 = 0; c0 < CHUNKS; c0 += G) {
    float4 t[G];
#pragma unroll
    for (int c = 0; c < G; ++c) t[c] = xr[(c0 + c) * 32 + lane];
#pragma unroll
    for (int c = 0; c < G; ++c) {
      const uint2 wu = wr[(c0 + c) * 32 + lane];
      const float2 w01 = unpack_bf2(wu.x), w23 = unpack_bf2(wu.y);
      uint2 o;
      o.x = pack_bf2(w01.x * (round_bf(t[c].x) * inv), w01.y * (round_bf(t[c].y) * inv));
      o.y = pack_bf2(w23.x * (round_bf(t[c].z) * inv), w23.y * (round_bf(t[c].w) * inv));
      orow[(c0 + c) * 32 + lane] = o;
      if (trow) trow[(c0 + c) * 32 + lane] = o;
    }
  }
}

// The same norm with one 128-thread CTA per row (H = 512 * V): every thread
// holds its V float4 of the row in registers, so the row is read once and
// the kernel makes one dependent round trip to memory per row (the
// warp-per-row form above makes four); up to 16 rows are in flight per SM.
template <int V>
__global__ void __launch_bounds__(128) rmsnorm_row_kernel(const float* __restrict__ x, int row_mul, int row_add,
                                                          const __nv_bfloat16* __restrict__ w,
                                                          __nv_bfloat16* __restrict__ out,
                                                          __nv_bfloat16* __restrict__ tap, int M, float eps,
                                                          const __nv_bfloat16* __restrict__ copy_src, int n_copy) {
  constexpr int H = 512 * V;
  __shared__ float red[4];
  griddep_begin();
  const int row = blockIdx.x, t = threadIdx.x;
  if (row >= M) {  // verbatim copy rows (decode: prev_hs feeds the delayed values)
    const uint2* src = reinterpret_cast<const uint2*>(copy_src + (size_t)(row - M) * H);
    uint2* dst = reinterpret_cast<uint2*>(out + (size_t)row * H);
#pragma unroll
    for (int c = 0; c < V; ++c) dst[c * 128 + t] = src[c * 128 + t];
    return;
  }
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)(row * row_mul + row_add) * H);
  const uint2* wr = reinterpret_cast<const uint2*>(w);
  float4 v[V];
  uint2 wu[V];
#pragma unroll
  for (int c = 0; c < V; ++c) {
    v[c] = xr[c * 128 + t];
    wu[c] = __ldg(wr + c * 128 + t);
  }
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < V; ++c) {
    v[c] = make_float4(round_bf(v[c].x), round_bf(v[c].y), round_bf(v[c].z), round_bf(v[c].w));
    ss += v[c].x * v[c].x + v[c].y * v[c].y + v[c].z * v[c].z + v[c].w * v[c].w;
  }
  ss = warp_sum(ss);
  if (lane_id() == 0) red[warp_id()] = ss;
  __syncthreads();
  const float inv = rsqrtf(((red[0] + red[1]) + (red[2] + red[3])) / (float)H + eps);
  uint2* orow = reinterpret_cast<uint2*>(out + (size_t)row * H);
  uint2* trow = tap ? reinterpret_cast<uint2*>(tap + (size_t)row * H) : nullptr;
#pragma unroll
  for (int c = 0; c < V; ++c) {
    const float2 w01 = unpack_bf2(wu[c].x), w23 = unpack_bf2(wu[c].y);
    uint2 o;
    o.x = pack_bf2(w01.x * (v[c].x * inv), w01.y * (v[c].y * inv));
    o.y = pack_bf2(w23.x * (v[c].z * inv), w23.y * (v[c].w * inv));
    orow[c * 128 + t] = o;
    if (trow) trow[c * 128 + t] = o;
  }
}

// stream[m] = fp32((E[id] + shift) * mult); one warp per row.
__global__ void __launch_bounds__(256) embed_kernel(const int* __restrict__ ids, const __nv_bfloat16* __restrict__ table,
                                                    float* __restrict__ stream, int M, int H, int vocab, float mult,
                                                    float shift, int* status) {
  griddep_begin();
  const int row = blockIdx.x * 8 + warp_id();
  const int lane = lane_id();
  if (row >= M) return;
  const int id = ids[row];
  float4* dst = reinterpret_cast<float4*>(stream + (size_t)row * H);
  if (id < 0 || id >= vocab) {
    if (lane == 0) set_status(status, ZAYA_ERR_DEVICE_RANGE);
    for (int c = lane; c < H / 4; c += 32) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const uint2* src = reinterpret_cast<const uint2*>(table + (size_t)id * H);
  for (int c = lane; c < H / 4; c += 32) {
    const uint2 u = src[c];
    const float2 a = unpack_bf2(u.x), b = unpack_bf2(u.y);
    dst[c] = make_float4((a.x + shift) * mult, (a.y + shift) * mult, (b.x + shift) * mult, (b.y + shift) * mult);
  }
}

}  // namespace

int launch_rmsnorm(const float* x, int row_mul, int row_add, const void* w, void* out, void* tap, int M, int H,
                   float eps, const void* copy_src, int n_copy, cudaStream_t st) {
  const int rows = M + n_copy;
  if (rows <= 0) return ZAYA_OK;
  const auto* wb = static_cast<const __nv_bfloat16*>(w);
  auto* ob = static_cast<__nv_bfloat16*>(out);
  auto* tb = static_cast<__nv_bfloat16*>(tap);
  const auto* cs = static_cast<const __nv_bfloat16*>(copy_src);
  const int v = H % 512 ? 0 : H / 512;   // one CTA per row when H is a multiple of 512
  if (v == 1 || v == 2 || v == 4 || v == 8) {
    cudaError_t e;
    if (v == 1) e = launch_k_as(0, rmsnorm_row_kernel<1>, dim3(rows), dim3(128), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy);
    else if (v == 2) e = launch_k_as(0, rmsnorm_row_kernel<2>, dim3(rows), dim3(128), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy);
    else if (v == 4) e = launch_k_as(0, rmsnorm_row_kernel<4>, dim3(rows), dim3(128), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy);
    else e = launch_k_as(0, rmsnorm_row_kernel<8>, dim3(rows), dim3(128), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy);
    return e == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
  }
  const dim3 grid((rows + 7) / 8);
  switch (H / 128) {
    case 2: launch_k_as(0, rmsnorm_kernel<2>, grid, dim3(256), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy); break;
    case 4: launch_k_as(0, rmsnorm_kernel<4>, grid, dim3(256), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy); break;
    case 8: launch_k_as(0, rmsnorm_kernel<8>, grid, dim3(256), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy); break;
    case 16: launch_k_as(0, rmsnorm_kernel<16>, grid, dim3(256), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy); break;
    case 32: launch_k_as(0, rmsnorm_kernel<32>, grid, dim3(256), 0, st, nullptr, 0, x, row_mul, row_add, wb, ob, tb, M, eps, cs, n_copy); break;
    default: return ZAYA_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

int launch_embed(const int* ids, const void* table, float* stream, int M, int H, int vocab, float mult, float shift,
                 int* status, cudaStream_t st) {
  if (M <= 0) return ZAYA_OK;
  launch_k(embed_kernel, dim3((M + 7) / 8), dim3(256), 0, st, nullptr, 0, ids,
           static_cast<const __nv_bfloat16*>(table), stream, M, H, vocab, mult, shift, status);
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

}  // namespace zaya
