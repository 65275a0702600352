// tcgen05 GEMM for the ZAYA1 block's dense contractions (sm_100a).
//
// C[M, N] = A[M, K] * B[N, K]^T with bf16 operands and fp32 accumulation in
// tensor memory.  One persistent CTA per SM walks 128 x BN output tiles:
//   warp 0      TMA producer: 128x64 A and BNx64 B tiles into a STAGES-deep
//               shared-memory ring (128-byte swizzle), one mbarrier per slot;
//   warp 1      one elected thread issues tcgen05.mma (M=128, N=BN, K=16) into
//               one of two TMEM accumulators and commits slot releases;
//   warps 2..   epilogue (4 warps; 8 for the merge epilogues, two per TMEM
//               lane quarter splitting the columns): tcgen05.ld of the finished
//               accumulator (each warp reads the 32 TMEM lanes its warp index
//               allows), the fused epilogue, global stores; then the
//               accumulator is handed back, so the epilogue of tile i overlaps
//               the main loop of tile i+1.
// The producer also pulls B (weight) boxes into L2 eight k-blocks ahead of
// their loads, so the ring's loads wait on L2 rather than on HBM.
// Grouped mode (the experts): A rows are the tokens permuted by expert, B is
// the stacked expert weights; the tile list is derived on the device from
// the per-expert row offsets, so no host synchronisation is needed.
// Grouped CTA pairs run swapped (D^T = W X^T): the expert's weight rows are
// the MMA's M = 256 side and its tokens the N side, N = the tile's token count
// rounded up to 16 (an expert's tokens split into ceil(n/256) near-equal
// tiles), so a routed token costs 1/16 of padding at most instead of up to a
// whole 256-row tile.  The epilogue then holds one feature per TMEM lane and
// one token per column.
//
// Epilogues (what the block needs right after each contraction):
//   STORE_BF16   q/k/v projections, lm_head logits
//   MERGE_ATTN   o_proj, then merge 1 of the zaya page ("The block, in
//                order"): attention_output = bf16((o + hb) * hs);
//                h = attention_output + (x + rb) * rs written over x
//   ROUTER_DOWN  router down_proj + bias + previous state * router_states_scale
//   STORE_F32    fp32 partial sums of a split-K product (router down_proj: the
//                router kernel adds the slabs in a fixed order)
//   SWIGLU       expert gate/up: act = bf16(silu(gate) * up)
//   MERGE_MLP    expert down: y = w_t * acc; mlp_output = bf16((y + hb) * hs);
//                out = mlp_output + (h + rb) * rs, scattered to token t's row
#include <stdio.h>

#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_STAGE_BYTES = BM * BK * 2;

template <int EPI>
__host__ __device__ constexpr int epi_warps() { return (EPI == EPI_MERGE_ATTN || EPI == EPI_MERGE_MLP) ? 8 : 4; }
template <int EPI>
__host__ __device__ constexpr bool is_merge() { return EPI == EPI_MERGE_ATTN || EPI == EPI_MERGE_MLP; }
constexpr int kPrefetchAhead = 8;  // k-blocks of B pulled into L2 ahead of their TMA load

constexpr int kSmemLimit = 232448;  // dynamic shared memory per CTA (227 KB)

template <int BN, int EPI, int CG = 1, bool SWAP = false>
struct GemmCfg {
  static constexpr int B_STAGE_BYTES = BN / CG * BK * 2;   // a CTA pair splits B's columns (swapped: 128 token rows)
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulators
  // merge: [2 tiles][hb,hs,rb,rs][BN] fp32 (swapped: per-lane registers instead)
  static constexpr int PARAM_BYTES = (is_merge<EPI>() && !SWAP) ? 2 * 4 * BN * 4 : 0;
  // merge epilogues: a 32 x 32 fp32 transpose buffer per epilogue warp; swapped
  // SwiGLU: per chunk two feature groups x (16 gate + 16 up tokens) x 32 lanes, double-buffered
  static constexpr int T_BYTES = (SWAP && EPI == EPI_SWIGLU) ? 2 * 2 * 32 * 32 * 4
                                 : (is_merge<EPI>() ? epi_warps<EPI>() * 32 * 32 * 4 : 0);
  static constexpr int FIXED = PARAM_BYTES + T_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr int DEF_STAGES = (STAGE_BYTES >= 49152) ? 4 : (STAGE_BYTES >= 32768 ? 6 : 8);  // ~192 KB ring
  static constexpr int FIT_STAGES = (kSmemLimit - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = DEF_STAGES < FIT_STAGES ? DEF_STAGES : FIT_STAGES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED;
  static_assert(STAGES >= 3, "ring too shallow");
};

struct TileInfo {
  int kb0;     // first k-block of this tile's K slab
  int nkb;     // k-blocks in the slab
  int split;   // slab index (STORE_F32)
  int m0;      // first A row
  int m_end;   // A rows of this tile's group end here (exclusive)
  int n0;      // first output column
  int b_row;   // first B row (gate rows for SWIGLU)
  int b_row2;  // SWIGLU: first up row
  int n_valid; // swapped: the tile's tokens (rows m0 .. m0 + n_valid of A)
  int n_mma;   // swapped: MMA N, n_valid rounded up to 16
  int e;       // grouped: the expert
};

template <int EPI, int BN_OUT, int TM>   // TM: output rows per tile (128, or 256 for a CTA pair)
__device__ __forceinline__ int total_tiles(const GemmParams& p) {
  const int nt = p.N / BN_OUT;
  const int ks = p.k_splits > 1 ? p.k_splits : 1;
  if (!p.grouped) return ((p.M + TM - 1) / TM) * nt * ks;
  return p.mt_start[p.n_groups] * nt;   // mt_start counts TM-row tiles
}

// KE: K elements per k-block (a 128-byte smem row: 64 bf16, 128 E4M3)
template <int EPI, int BN_OUT, int TM, bool SWAP = false, int KE = BK>
__device__ __forceinline__ TileInfo tile_info(const GemmParams& p, int t) {
  TileInfo ti;
  const int nt = p.N / BN_OUT;
  const int ks = p.k_splits > 1 ? p.k_splits : 1;
  ti.nkb = p.K / KE / ks;
  ti.e = 0;
  ti.split = 0;
  ti.kb0 = 0;
  if (!p.grouped) {
    const int mt = (p.M + TM - 1) / TM;
    ti.m0 = (t % mt) * TM;
    const int rest = t / mt;
    ti.split = rest % ks;
    ti.kb0 = ti.split * ti.nkb;
    ti.n0 = (rest / ks) * BN_OUT;
    ti.m_end = p.M;
    ti.b_row = ti.n0;
    ti.b_row2 = ti.n0;
  } else {
    int e = 0;
    while (e + 1 < p.n_groups && p.mt_start[e + 1] * nt <= t) ++e;
    const int local = t - p.mt_start[e] * nt;
    const int mte = p.mt_start[e + 1] - p.mt_start[e];
    ti.m0 = p.group_off[e] + (local % mte) * TM;
    ti.m_end = p.group_off[e + 1];
    ti.n0 = (local / mte) * BN_OUT;
    ti.b_row = e * p.b_rows_per_group + ti.n0;
    ti.b_row2 = e * p.b_rows_per_group + (p.b_rows_per_group >> 1) + ti.n0;
    ti.e = e;
    if constexpr (SWAP) {
      // the expert's n tokens in mte near-equal tiles of `per` (a multiple of 16,
      // at most 256); every tile holds at least one token since n > 256 (mte - 1)
      const int n = ti.m_end - p.group_off[e];
      const int per = ((n + mte - 1) / mte + 15) & ~15;
      const int i = local % mte;
      ti.m0 = p.group_off[e] + i * per;
      ti.n_valid = min(per, n - i * per);
      ti.n_mma = (ti.n_valid + 15) & ~15;
    }
  }
  return ti;
}

// silu(g) = g / (1 + e^-g) with the fast (branch-free) division: a few ulp in
// fp32 ahead of the bf16 rounding of act, and no per-element branch that would
// serialise the epilogue's chains (g -> -inf gives -0).
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Epilogue of one row (this thread) x 32 consecutive columns.
template <int EPI>
__device__ __forceinline__ void epilogue32(const GemmParams& p, int row, int col, int split, const uint32_t (&r)[32],
                                           const uint32_t (&r2)[32], const float* prm, int prm_ld) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  if constexpr (EPI == EPI_STORE_BF16 || EPI == EPI_SWIGLU) {
    if constexpr (EPI == EPI_SWIGLU) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = silu_f(v[j]) * __uint_as_float(r2[j]);
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + (size_t)row * p.ldo + col);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u;
      u.x = pack_bf2(v[8 * q + 0], v[8 * q + 1]);
      u.y = pack_bf2(v[8 * q + 2], v[8 * q + 3]);
      u.z = pack_bf2(v[8 * q + 4], v[8 * q + 5]);
      u.w = pack_bf2(v[8 * q + 6], v[8 * q + 7]);
      dst[q] = u;
    }
  } else if constexpr (EPI == EPI_STORE_F32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + ((size_t)split * p.M + row) * p.ldo + col);
#pragma unroll
    for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else if constexpr (EPI == EPI_ROUTER_DOWN) {
    float* dst = static_cast<float*>(p.out) + (size_t)row * p.ldo + col;
    const float* prev = p.prev ? p.prev + (size_t)row * p.N + col : nullptr;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 o;
      float* op = &o.x;
      float4 pv = prev ? *reinterpret_cast<const float4*>(prev + 4 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float* pp = &pv.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = col + 4 * q + j;
        float x = v[4 * q + j] + __ldg(p.bias + c);
        if (prev) x = fmaf(pp[j], __ldg(p.prev_scale + c), x);
        op[j] = x;
      }
      reinterpret_cast<float4*>(dst)[q] = o;
    }
  } else {  // MERGE_ATTN / MERGE_MLP
    int token = row;
    float wt = 1.0f;
    if constexpr (EPI == EPI_MERGE_MLP) {
      token = p.perm[row];
      wt = p.row_w[token];
    }
    const int N = p.N;
    float* srow = p.stream + (size_t)token * N + col;
    __nv_bfloat16* tap = p.tap_bf16 ? static_cast<__nv_bfloat16*>(p.tap_bf16) + (size_t)token * N + col : nullptr;
    float* tapf = p.tap_f32 ? p.tap_f32 + (size_t)token * N + col : nullptr;
    float4 xs[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) xs[q] = reinterpret_cast<const float4*>(srow)[q];   // all loads in flight first
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 x4 = xs[q];
      float* xp = &x4.x;
      const float4 hb4 = *reinterpret_cast<const float4*>(prm + 4 * q);
      const float4 hs4 = *reinterpret_cast<const float4*>(prm + prm_ld + 4 * q);
      const float4 rb4 = *reinterpret_cast<const float4*>(prm + 2 * prm_ld + 4 * q);
      const float4 rs4 = *reinterpret_cast<const float4*>(prm + 3 * prm_ld + 4 * q);
      const float* hbp = &hb4.x;
      const float* hsp = &hs4.x;
      const float* rbp = &rb4.x;
      const float* rsp = &rs4.x;
      float cb[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float contrib = round_bf((v[4 * q + j] * wt + hbp[j]) * hsp[j]);
        cb[j] = contrib;
        xp[j] = fmaf(xp[j] + rbp[j], rsp[j], contrib);
      }
      reinterpret_cast<float4*>(srow)[q] = x4;
      if (tapf) reinterpret_cast<float4*>(tapf)[q] = x4;
      if (tap) {
        uint2 u;
        u.x = pack_bf2(cb[0], cb[1]);
        u.y = pack_bf2(cb[2], cb[3]);
        reinterpret_cast<uint2*>(tap)[q] = u;
      }
    }
  }
}

// Merge epilogue of a warp's 32 rows x 32 columns, coalesced: the accumulator
// rows (one per lane, as tcgen05.ld delivers them) go through a 32 x 32 fp32
// shared-memory transpose (16-byte chunks XOR-swizzled by row), then each
// step covers 4 rows x 128 contiguous bytes of the fp32 stream; all eight
// steps' stream loads are issued before the first use.
template <int EPI>
__device__ __forceinline__ void merge_chunk(const GemmParams& p, int row0, int m_end, int col,
                                            const uint32_t (&r)[32], float* T, const float* prm, int prm_ld) {
  const int lane = lane_id();
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4*>(T + lane * 32 + ((j ^ (lane & 7)) << 2)) =
        make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]), __uint_as_float(r[4 * j + 2]),
                    __uint_as_float(r[4 * j + 3]));
  __syncwarp();
  const int jj = lane & 7, rsub = lane >> 3;
  const int N = p.N;
  int tok[8];
  float wt[8];
  float4 xs[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int grow = row0 + 4 * i + rsub;
    tok[i] = -1;
    if (grow < m_end) tok[i] = (EPI == EPI_MERGE_MLP) ? p.perm[grow] : grow;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    wt[i] = 1.0f;
    xs[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tok[i] >= 0) {
      if constexpr (EPI == EPI_MERGE_MLP) wt[i] = p.row_w[tok[i]];
      xs[i] = *reinterpret_cast<const float4*>(p.stream + (size_t)tok[i] * N + col + 4 * jj);
    }
  }
  const float4 hb4 = *reinterpret_cast<const float4*>(prm + 4 * jj);
  const float4 hs4 = *reinterpret_cast<const float4*>(prm + prm_ld + 4 * jj);
  const float4 rb4 = *reinterpret_cast<const float4*>(prm + 2 * prm_ld + 4 * jj);
  const float4 rs4 = *reinterpret_cast<const float4*>(prm + 3 * prm_ld + 4 * jj);
  const float* hbp = &hb4.x;
  const float* hsp = &hs4.x;
  const float* rbp = &rb4.x;
  const float* rsp = &rs4.x;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (tok[i] < 0) continue;
    const int rr = 4 * i + rsub;
    const float4 a4 = *reinterpret_cast<const float4*>(T + rr * 32 + ((jj ^ (rr & 7)) << 2));
    const float* ap = &a4.x;
    float4 x4 = xs[i];
    float* xp = &x4.x;
    float cb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float contrib = round_bf((ap[j] * wt[i] + hbp[j]) * hsp[j]);
      cb[j] = contrib;
      xp[j] = fmaf(xp[j] + rbp[j], rsp[j], contrib);
    }
    const size_t off = (size_t)tok[i] * N + col + 4 * jj;
    *reinterpret_cast<float4*>(p.stream + off) = x4;
    if (p.tap_f32) *reinterpret_cast<float4*>(p.tap_f32 + off) = x4;
    if (p.tap_bf16) {
      uint2 u;
      u.x = pack_bf2(cb[0], cb[1]);
      u.y = pack_bf2(cb[2], cb[3]);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.tap_bf16) + off) = u;
    }
  }
  __syncwarp();
}

// Swapped merge epilogue of a warp's 32 features (lanes, from fw) x 32
// permuted rows (columns, from row0; nj of them real): the accumulator goes
// through a 32 x 32 fp32 shared-memory transpose to token-major 16-byte chunks
// (XOR-swizzled by token), then each step covers 4 tokens x 128 contiguous
// bytes of the fp32 stream, all eight steps' loads in flight first.  tokl /
// wl: lane i holds row row0 + i's token and routing weight.
__device__ __forceinline__ void merge_chunk_swap(const GemmParams& p, int nj, int fw, int tokl, float wl,
                                                 const uint32_t (&r)[32], float* T, const float4* dsc) {
  const int lane = lane_id();
#pragma unroll
  for (int j = 0; j < 32; ++j) T[j * 32 + (((lane >> 2) ^ (j & 7)) << 2) + (lane & 3)] = __uint_as_float(r[j]);
  __syncwarp();
  const int jj = lane & 7, rsub = lane >> 3;
  const int N = p.N;
  const int col = fw + 4 * jj;
  int tok[8];
  float wt[8];
  float4 xs[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    tok[i] = __shfl_sync(0xffffffffu, tokl, 4 * i + rsub);
    wt[i] = __shfl_sync(0xffffffffu, wl, 4 * i + rsub);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
    xs[i] = 4 * i + rsub < nj ? *reinterpret_cast<const float4*>(p.stream + (size_t)tok[i] * N + col)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 hb4 = __ldg(reinterpret_cast<const float4*>(p.merge + col));
  const float4 hs4 = __ldg(reinterpret_cast<const float4*>(p.merge + N + col));
  const float4 rb4 = __ldg(reinterpret_cast<const float4*>(p.merge + 2 * N + col));
  const float4 rs4 = __ldg(reinterpret_cast<const float4*>(p.merge + 3 * N + col));
  const float* hbp = &hb4.x;
  const float* hsp = &hs4.x;
  const float* rbp = &rb4.x;
  const float* rsp = &rs4.x;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = 4 * i + rsub;
    if (rr >= nj) continue;
    float4 a4 = *reinterpret_cast<const float4*>(T + rr * 32 + ((jj ^ (rr & 7)) << 2));
    if (dsc) {   // E4M3 products: s_act times the rows' scales
      a4.x *= dsc->x; a4.y *= dsc->y; a4.z *= dsc->z; a4.w *= dsc->w;
    }
    const float* ap = &a4.x;
    float4 x4 = xs[i];
    float* xp = &x4.x;
    float cb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float contrib = round_bf((ap[j] * wt[i] + hbp[j]) * hsp[j]);
      cb[j] = contrib;
      xp[j] = fmaf(xp[j] + rbp[j], rsp[j], contrib);
    }
    const size_t off = (size_t)tok[i] * N + col;
    *reinterpret_cast<float4*>(p.stream + off) = x4;
    if (p.tap_bf16) {
      uint2 u;
      u.x = pack_bf2(cb[0], cb[1]);
      u.y = pack_bf2(cb[2], cb[3]);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.tap_bf16) + off) = u;
    }
  }
  __syncwarp();
}

// CG = 1: one CTA per SM, 128 x BN tiles.  CG = 2: clusters of two CTAs
// (cta_group::2), 256 x BN tiles: CTA rank r loads A rows [m0 + 128r, +128)
// and its half of B's BN rows (SWIGLU: rank 0 the gate rows, rank 1 the up
// rows), both completing on the rank-0 CTA's `full` barrier, whose producer
// alone arms it with both CTAs' bytes; rank 0's MMA thread issues M = 256
// MMAs and its commits arrive on the `empty` / `tfull` barriers of both CTAs;
// each CTA's epilogue reads its own 128 accumulator rows and releases the
// accumulator on rank 0's `tempty`.
// SWAP (grouped CTA pairs): CTA rank r loads 128 weight rows into the A slot
// (SWIGLU: gate rows [n0 + 64r, +64) then the up rows of the same features;
// MERGE_MLP: output rows [n0 + 128r, +128)) and its n_mma / 2 token rows from
// m0 + r * n_mma / 2 into the B slot, in boxes of tok_box (16) rows, so a
// tile of few tokens loads few bytes; tmA then maps the tokens and tmB the
// weights.
// F8 (swapped only): E4M3 operands on kind::f8f6f4, a k-block is 128 elements
// (the same 128-byte rows), and the epilogues apply the static input scale
// and the per-row weight scale of the expert (the SwiGLU output is stored as
// E4M3 codes of act / s_act for the down projection).
template <int BN, int EPI, int CG, bool SWAP, bool F8 = false>
__global__ void __launch_bounds__(64 + 32 * epi_warps<EPI>(), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
  static_assert(!SWAP || (CG == 2 && BN == 256 && (EPI == EPI_SWIGLU || EPI == EPI_MERGE_MLP)),
                "swapped tiles: grouped expert GEMMs on CTA pairs");
  static_assert(!F8 || SWAP, "E4M3 operands: swapped expert tiles only");
  constexpr int KE = F8 ? 2 * BK : BK;   // K elements per k-block
  using C = GemmCfg<BN, EPI, CG, SWAP>;
  constexpr int STAGES = C::STAGES;
  constexpr int BN_OUT = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
  constexpr int TM = BM * CG;   // output rows per tile
  constexpr uint32_t IDESC = idesc_bf16_f32(TM, BN);
  constexpr int EW = epi_warps<EPI>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
  float* sPrm = reinterpret_cast<float*>(sB + STAGES * C::B_STAGE_BYTES);   // merge params [2][4][BN_OUT]
  float* sT = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sPrm) + C::PARAM_BYTES);   // [EW][32][32]
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sT) + C::T_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mdrain = tempty + 2;   // the MMA thread's last commit: all its MMAs are done
  uint64_t* xbar = mdrain + 1;     // [2] swapped SwiGLU: a chunk's gate / up halves are in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 2);
  int* s_skip = reinterpret_cast<int*>(tmem_slot + 1);   // CTA pair: rank 0's reading of the status word

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const int unit = (CG == 2) ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;   // tile walker index
  const int n_units = (CG == 2) ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], CG * EW);
    }
    mbar_init(mdrain, 1);
    mbar_init(&xbar[0], EW);
    mbar_init(&xbar[1], EW);
    fence_barrier_init();
    fence_proxy_async();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    if constexpr (CG == 2) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    else tmem_alloc(tmem_slot, C::TMEM_COLS);
  }
  tc_fence_before();
  __syncwarp();
  if constexpr (CG == 2) cluster_sync_all();   // both CTAs' barriers and TMEM are ready
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The prologue above (with the tensor-memory allocation) overlaps the
  // previous kernel, and is complete in every warp before any thread lets the
  // next kernel launch.  Global memory only from here.  A fault already
  // recorded in the status word (an earlier wait ran out) means the launch
  // chain has failed: the kernel then does no work.  Both CTAs of a pair take
  // rank 0's reading, so that they walk the same tiles.
  griddep_begin();
  WaitCtx wc = wait_ctx(p.status, /*bail=*/CG == 1);
  if constexpr (CG == 2) {
    if (rank == 0 && threadIdx.x == 0) {
      const uint32_t v = wc.skip ? 1u : 0u;
      *s_skip = v;
      asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa_shared(s_skip, 1)), "r"(v) : "memory");
    }
    cluster_sync_all();   // rank 0's reading is published to both CTAs
    wc.skip = *reinterpret_cast<volatile int*>(s_skip) != 0;
  }

  const int ntiles = wc.skip ? 0 : total_tiles<EPI, BN_OUT, TM>(p);

  if (warp == 0) {
    // ---------------- TMA producer (each CTA loads its own A rows and B half)
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int n_armed = 0;
      for (int t = unit; t < ntiles; t += n_units) {
        const TileInfo ti = tile_info<EPI, BN_OUT, TM, SWAP, KE>(p, t);
        // this CTA's B rows: CG = 1 all BN rows (SWIGLU: gate then up); CG = 2 its half
        const int b_first = (CG == 1) ? ti.b_row
                            : SWAP ? ti.b_row + (int)rank * (EPI == EPI_SWIGLU ? 64 : 128)
                            : (EPI == EPI_SWIGLU) ? (rank == 0 ? ti.b_row : ti.b_row2)
                                                  : ti.b_row + (int)rank * (BN / 2);
        const int kb_end = ti.kb0 + ti.nkb;
        auto prefetch_b = [&](int kb) {
          if constexpr (SWAP && EPI == EPI_SWIGLU) {
            tma_prefetch_l2_2d(&tmB, kb * KE, b_first);
            tma_prefetch_l2_2d(&tmB, kb * KE, ti.b_row2 + (int)rank * 64);
          } else if constexpr (EPI == EPI_SWIGLU && CG == 1) {
            tma_prefetch_l2_2d(&tmB, kb * KE, ti.b_row);
            tma_prefetch_l2_2d(&tmB, kb * KE, ti.b_row2);
          } else {
            tma_prefetch_l2_2d(&tmB, kb * KE, b_first);
          }
        };
        for (int kb = ti.kb0; kb < ti.kb0 + kPrefetchAhead && kb < kb_end; ++kb) prefetch_b(kb);
        for (int kb = ti.kb0; kb < kb_end; ++kb) {
          if (kb + kPrefetchAhead < kb_end) prefetch_b(kb + kPrefetchAhead);
          if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) goto producer_done;
          uint8_t* a_dst = sA + stage * A_STAGE_BYTES;
          uint8_t* b_dst = sB + stage * C::B_STAGE_BYTES;
          if constexpr (SWAP) {
            // tokens: the n_mma / 2 rows of this CTA's half of N, in boxes of tok_box rows
            const int n_box = ((ti.n_mma >> 1) + p.tok_box - 1) / p.tok_box;
            if (rank == 0)   // both CTAs' bytes
              mbar_arrive_expect_tx(&full[stage], 2 * (A_STAGE_BYTES + n_box * p.tok_box * BK * 2));
            const uint32_t bar = mapa_shared(&full[stage], 0);
            tma_load_2d_pair(a_dst, &tmB, bar, kb * KE, b_first);   // weights: the MMA's A
            if constexpr (EPI == EPI_SWIGLU)
              tma_load_2d_pair(a_dst + 64 * BK * 2, &tmB, bar, kb * KE, ti.b_row2 + (int)rank * 64);
            const int t0 = ti.m0 + (int)rank * (ti.n_mma >> 1);
            for (int bx = 0; bx < n_box; ++bx)
              tma_load_2d_pair(b_dst + bx * p.tok_box * BK * 2, &tmA, bar, kb * KE, t0 + bx * p.tok_box);
          } else if constexpr (CG == 2) {
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);   // both CTAs' bytes
            const uint32_t bar = mapa_shared(&full[stage], 0);
            tma_load_2d_pair(a_dst, &tmA, bar, kb * KE, ti.m0 + (int)rank * BM);
            tma_load_2d_pair(b_dst, &tmB, bar, kb * KE, b_first);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
            tma_load_2d(a_dst, &tmA, &full[stage], kb * KE, ti.m0);
            if constexpr (EPI == EPI_SWIGLU) {
              tma_load_2d(b_dst, &tmB, &full[stage], kb * KE, ti.b_row);
              tma_load_2d(b_dst + (BN / 2) * BK * 2, &tmB, &full[stage], kb * KE, ti.b_row2);
            } else {
              tma_load_2d(b_dst, &tmB, &full[stage], kb * KE, ti.b_row);
            }
          }
          ++n_armed;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      // Before the CTA may exit, every copy this producer started has landed:
      // wait for the last phase it armed on each slot (rank 0 arms both CTAs'
      // bytes of a pair, so its wait covers the peer's copies too).
      if (CG == 1 || rank == 0) {
        for (int s2 = 0; s2 < STAGES && s2 < n_armed; ++s2)
          mbar_drain(&full[s2], (s2 < stage) ? phase : (phase ^ 1u), p.status);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (rank 0 of a pair issues for both CTAs)
    if (rank == 0 && elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int t = unit; t < ntiles; t += n_units, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const TileInfo ti = tile_info<EPI, BN_OUT, TM, SWAP, KE>(p, t);
        const int nkb = ti.nkb;
        const uint32_t idesc = F8 ? idesc_e4m3_f32(TM, ti.n_mma) : SWAP ? idesc_bf16_f32(TM, ti.n_mma) : IDESC;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            if constexpr (F8)
              tc_mma_e4m3_pair(d_tmem, smem_desc_k128(a_addr + k * 32), smem_desc_k128(b_addr + k * 32), idesc,
                               (kb | k) != 0 ? 1u : 0u);
            else if constexpr (CG == 2)
              tc_mma_bf16_pair(d_tmem, smem_desc_k128(a_addr + k * 32), smem_desc_k128(b_addr + k * 32), idesc,
                               (kb | k) != 0 ? 1u : 0u);
            else
              tc_mma_bf16(d_tmem, smem_desc_k128(a_addr + k * 32), smem_desc_k128(b_addr + k * 32), IDESC,
                          (kb | k) != 0 ? 1u : 0u);
          }
          if constexpr (CG == 2) tc_commit_pair(&empty[stage], 3);
          else tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (CG == 2) tc_commit_pair(&tfull[acc], 3);
        else tc_commit(&tfull[acc]);
      }
      // last commit: once it arrives every MMA of this thread has completed,
      // so the tensor memory may be freed
      if constexpr (CG == 2) tc_commit_pair(mdrain, 1);
      else tc_commit(mdrain);
      mbar_drain(mdrain, 0, p.status);
    }
  } else if constexpr (SWAP) {
    // ---------------- epilogue warps, swapped tiles: TMEM lane = weight row, column = token
    const int q = warp & 3;              // TMEM lanes [32q, 32q+32) are reachable from this warp
    const int part = (warp - 2) >> 2;    // MERGE_MLP: column interleave of the two warps per lane quarter
    const int N = p.N;
    int local = 0;
    uint32_t kc = 0;        // SWIGLU: chunks done, the parity of the up-value buffer
    bool aborted = false;   // a wait ran out: keep walking the tiles (barrier partners) without waiting
    for (int t = unit; t < ntiles; t += n_units, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const TileInfo ti = tile_info<EPI, BN_OUT, TM, SWAP, KE>(p, t);
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      if constexpr (EPI == EPI_SWIGLU) {
        // Lanes 0-63 hold the gate rows of features n0 + 64 rank + [0, 64), lanes
        // 64-127 their up rows.  Per 32-token chunk, warp q works on feature
        // group q & 1 and token half q >> 1: the gate warp hands its second
        // half of gate values to the up warp of its group and takes the up
        // warp's first half of up values (shared memory), then each warp writes
        // act = bf16(silu(gate) * up) for its 16 tokens x 32 features.
        // The hand-over of chunk kc completes xbar[kc & 1] (one arrival per warp)
        // for the (kc >> 1)-th time; a warp writes that buffer again two chunks
        // later, after the hand-over in between has completed, i.e. after
        // every warp has read it.  All waits are bounded: a warp that gives up
        // leaves the others to give up at their next hand-over.
        if (!aborted && !__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, wc))) aborted = true;
        if (aborted) continue;
        tc_fence_after();
        const int fg = q & 1, th = q >> 1;
        const int feat = ti.n0 + 64 * (int)rank + 32 * fg + lane;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
        // F8: the gate / up accumulators times s_in and their rows' scales; act
        // leaves as E4M3 codes of act / s_act
        float sg = 1.f, su = 1.f, inv_act = 1.f;
        if constexpr (F8) {
          const float s_in = __ldg(p.act_scale + 2 * ti.e);
          sg = s_in * __ldg(p.w_scale + (size_t)ti.e * p.b_rows_per_group + feat);
          su = s_in * __ldg(p.w_scale + (size_t)ti.e * p.b_rows_per_group + (p.b_rows_per_group >> 1) + feat);
          inv_act = __fdiv_rn(1.f, __ldg(p.act_scale + 2 * ti.e + 1));
        }
#pragma unroll 1
        for (int c = 0; c < ti.n_valid; c += 32, ++kc) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
          // [group][0: gate tokens 16-31 | 1: up tokens 0-15][16][32 lanes]
          float* T = sT + (kc & 1) * 2048 + fg * 1024;
          float* give = T + th * 512;    // gate warp gives gate (tokens 16-31), up warp gives up (tokens 0-15)
          float* take = T + (th ^ 1) * 512;
#pragma unroll
          for (int j = 0; j < 16; ++j) give[j * 32 + lane] = __uint_as_float(th == 0 ? r[j + 16] : r[j]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&xbar[kc & 1]);
          if (!__all_sync(0xffffffffu, mbar_wait(&xbar[kc & 1], (kc >> 1) & 1, wc))) {
            aborted = true;
            break;
          }
          float a[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float mine = __uint_as_float(th == 0 ? r[j] : r[j + 16]), other = take[j * 32 + lane];
            const float gate = (th == 0 ? mine : other) * sg, up = (th == 0 ? other : mine) * su;
            a[j] = silu_f(gate) * up;
          }
          const int j0 = c + 16 * th;
          const int nj = min(16, ti.n_valid - j0);
          if constexpr (F8) {
            uint8_t* dst8 = static_cast<uint8_t*>(p.out) + (size_t)(ti.m0 + j0) * p.ldo + feat;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j < nj) dst8[(size_t)j * p.ldo] = (uint8_t)(pack_e4m3x2(a[j] * inv_act, 0.f) & 0xffu);
          } else {
            __nv_bfloat16* dst = out + (size_t)(ti.m0 + j0) * p.ldo + feat;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j < nj) dst[(size_t)j * p.ldo] = __float2bfloat16_rn(a[j]);
          }
        }
        if (aborted) continue;
      } else {
        // MERGE_MLP: lane = output feature, column = permuted row; a token's 32
        // features of this warp are one 128-byte segment of its stream row.
        // While the main loop runs: this warp's chunks are columns 32 part + 64 k
        // (k < 4, N <= 256); lane j of chunk k fetches its token and routing
        // weight and pulls the token's stream segment into L2.
        const int fw = ti.n0 + 128 * (int)rank + 32 * q;   // this warp's first feature
        int tokk[4];
        float wk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int cc = 32 * part + 64 * k + lane;
          tokk[k] = cc < ti.n_valid ? p.perm[ti.m0 + cc] : 0;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const bool in = 32 * part + 64 * k + lane < ti.n_valid;
          wk[k] = in ? p.row_w[tokk[k]] : 0.f;
          if (in) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.stream + (size_t)tokk[k] * N + fw));
        }
        if (!aborted && !__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, wc))) aborted = true;
        if (aborted) continue;
        tc_fence_after();
        float4 dsc;   // F8: s_act x the scales of this lane's four output rows (after the transpose)
        if constexpr (F8) {
          const float s_act = __ldg(p.act_scale + 2 * ti.e + 1);
          const float4 ws = __ldg(reinterpret_cast<const float4*>(p.w_scale + (size_t)ti.e * p.b_rows_per_group + fw +
                                                                  4 * (lane & 7)));
          dsc = make_float4(s_act * ws.x, s_act * ws.y, s_act * ws.z, s_act * ws.w);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = 32 * part + 64 * k;
          if (c >= ti.n_valid) break;   // warp-uniform
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
          merge_chunk_swap(p, min(32, ti.n_valid - c), fw, tokk[k], wk[k], r, sT + (warp - 2) * 1024,
                           F8 ? &dsc : nullptr);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty[acc], 0));
    }
  } else {
    // ---------------- epilogue warps 2 .. 2+EW-1 (this CTA's 128 accumulator rows)
    const int q = warp & 3;              // TMEM lanes [32q, 32q+32) are reachable from this warp
    const int part = (warp - 2) >> 2;    // column interleave among the warps sharing a lane quarter
    const int et = threadIdx.x - 64;     // epilogue thread index
    const int row_off = (int)rank * BM;  // this CTA's first row inside the tile
    int local = 0;
    bool aborted = false;   // a wait ran out: keep walking the tiles (barrier partners) without waiting
    for (int t = unit; t < ntiles; t += n_units, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const TileInfo ti = tile_info<EPI, BN_OUT, TM, SWAP, KE>(p, t);
      float* prm = sPrm + acc * 4 * BN_OUT;
      if constexpr (is_merge<EPI>()) {
        // this tile's merge parameters (hb, hs, rb, rs for its columns) into shared memory
        for (int i = et; i < 4 * BN_OUT; i += EW * 32) {
          const int r = i / BN_OUT, c = i % BN_OUT;
          prm[i] = __ldg(p.merge + (size_t)r * p.N + ti.n0 + c);
        }
        // pull this thread's stream segment into L2 while the main loop runs
        const int prow = ti.m0 + row_off + q * 32 + lane;
        if (part == 0 && prow < ti.m_end) {
          const int token = (EPI == EPI_MERGE_MLP) ? p.perm[prow] : prow;
          const char* base = reinterpret_cast<const char*>(p.stream + (size_t)token * p.N + ti.n0);
#pragma unroll
          for (int off = 0; off < BN_OUT * 4; off += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(base + off));
        }
        named_barrier_sync(1, EW * 32);
      }
      // warp-uniform: the TMEM loads below are .sync.aligned
      if (!aborted && !__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, wc))) aborted = true;
      if (aborted) continue;
      tc_fence_after();
      const int row = ti.m0 + row_off + q * 32 + lane;
      const bool valid = row < ti.m_end;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c = part * 32; c < BN_OUT; c += 32 * (EW / 4)) {
        uint32_t r[32], r2[32];
        tmem_ld32(tbase + c, r);
        if constexpr (EPI == EPI_SWIGLU) tmem_ld32(tbase + BN / 2 + c, r2);
        tmem_ld_wait();
        if constexpr (is_merge<EPI>())
          merge_chunk<EPI>(p, ti.m0 + row_off + q * 32, ti.m_end, ti.n0 + c, r, sT + (warp - 2) * 1024, prm + c,
                           BN_OUT);
        else if (valid)
          epilogue32<EPI>(p, row, ti.n0 + c, ti.split, r, r2, prm + c, BN_OUT);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (CG == 2) mbar_arrive_cluster(mapa_shared(&tempty[acc], 0));
        else mbar_arrive(&tempty[acc]);
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync_all();   // no CTA leaves while its peer may still touch it
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

template <int BN, int EPI, int CG, bool SWAP = false, bool F8 = false>
int launch_impl(const CUtensorMap& ma, const CUtensorMap& mb, const GemmParams& p, int ntiles_hint, int num_sms,
                cudaStream_t st) {
  using C = GemmCfg<BN, EPI, CG, SWAP>;
  auto kern = gemm_tc_kernel<BN, EPI, CG, SWAP, F8>;
  static bool attr_set = false;
  static int max_pairs = 0;   // co-resident CTA pairs (CG = 2)
  if (!attr_set) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return ZAYA_ERR_CUDA;
    attr_set = true;
    if (CG == 2) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * (num_sms / 2));
      cfg.blockDim = dim3(64 + 32 * epi_warps<EPI>());
      cfg.dynamicSmemBytes = C::SMEM_BYTES;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return ZAYA_ERR_CUDA;
      max_pairs = n;
    }
  }
  const int max_units = (CG == 2) ? max_pairs : num_sms;
  int units = ntiles_hint < max_units ? ntiles_hint : max_units;
  if (units < 1) units = 1;
  if constexpr (CG == 1) {
    if (launch_k(kern, dim3(units), dim3(64 + 32 * epi_warps<EPI>()), C::SMEM_BYTES, st, nullptr, 0, ma, mb, p) !=
        cudaSuccess)
      return ZAYA_ERR_CUDA;
  } else {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    if (launch_k(kern, dim3(2 * units), dim3(64 + 32 * epi_warps<EPI>()), C::SMEM_BYTES, st, attr, 1, ma, mb, p) !=
        cudaSuccess)
      return ZAYA_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

}  // namespace

// E4M3 bytes: a box of box_rows x 128 (one 128-byte swizzled row per row).
int make_tmap_u8(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return ZAYA_ERR_CUDA;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || cols % 16) return ZAYA_ERR_MISALIGNED;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ZAYA_OK : ZAYA_ERR_CUDA;
}

int make_tmap_bf16(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return ZAYA_ERR_CUDA;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (cols * 2) % 16) return ZAYA_ERR_MISALIGNED;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ZAYA_OK : ZAYA_ERR_CUDA;
}

int launch_gemm(int epi, int bn, const void* A, int a_rows, const void* B, int b_rows, const GemmParams& p,
                int num_sms, cudaStream_t st) {
  if (p.fp8) {   // E4M3 expert GEMMs: swapped CTA pairs only
    if (!p.grouped || !p.pair || bn != 256 || (epi != EPI_SWIGLU && epi != EPI_MERGE_MLP) || p.K % (2 * BK) ||
        p.K <= 0 || !p.w_scale || !p.act_scale)
      return ZAYA_ERR_UNSUPPORTED;
    if (p.N % (epi == EPI_SWIGLU ? bn / 2 : bn)) return ZAYA_ERR_UNSUPPORTED;
    if (a_rows <= 0) return ZAYA_OK;
    GemmParams q = p;
    q.tok_box = 16;
    CUtensorMap ma, mb;
    int rc = make_tmap_u8(&ma, A, (uint64_t)a_rows, (uint64_t)p.K, (uint32_t)q.tok_box);
    if (rc) return rc;
    rc = make_tmap_u8(&mb, B, (uint64_t)b_rows, (uint64_t)p.K, epi == EPI_SWIGLU ? 64 : 128);
    if (rc) return rc;
    return epi == EPI_SWIGLU ? launch_impl<256, EPI_SWIGLU, 2, true, true>(ma, mb, q, num_sms, num_sms, st)
                             : launch_impl<256, EPI_MERGE_MLP, 2, true, true>(ma, mb, q, num_sms, num_sms, st);
  }
  if (p.K % BK != 0 || p.K <= 0) return ZAYA_ERR_UNSUPPORTED;
  const int ks = p.k_splits > 1 ? p.k_splits : 1;
  if ((p.K / BK) % ks != 0 || (ks > 1 && (p.grouped || epi != EPI_STORE_F32))) return ZAYA_ERR_UNSUPPORTED;
  const int bn_out = (epi == EPI_SWIGLU) ? bn / 2 : bn;
  if (p.N % bn_out != 0) return ZAYA_ERR_UNSUPPORTED;
  if (a_rows <= 0) return ZAYA_OK;
  const int cg = p.pair ? 2 : 1;
  if (cg == 2 && bn != 256 && bn != 128) return ZAYA_ERR_UNSUPPORTED;
  // grouped expert GEMMs on CTA pairs run swapped (weights on the M side)
  const bool swap = cg == 2 && p.grouped && (epi == EPI_SWIGLU || epi == EPI_MERGE_MLP);
  if (swap && bn != 256) return ZAYA_ERR_UNSUPPORTED;
  // swapped: token boxes of 16 rows (two 128-byte swizzle atoms), as many as
  // a tile's half of N needs
  GemmParams q = p;
  q.tok_box = swap ? 16 : BM;
  CUtensorMap ma, mb;
  int rc = make_tmap_bf16(&ma, A, (uint64_t)a_rows, (uint64_t)p.K, (uint32_t)q.tok_box);
  if (rc) return rc;
  // B box: a CTA pair splits the tile's B rows in two; SWIGLU loads gate and up rows as two boxes
  // (swapped SWIGLU: 64 gate and 64 up rows per CTA)
  const uint32_t b_box = (swap && epi == EPI_SWIGLU) ? 64 : (epi == EPI_SWIGLU || cg == 2) ? bn / 2 : bn;
  rc = make_tmap_bf16(&mb, B, (uint64_t)b_rows, (uint64_t)p.K, b_box);
  if (rc) return rc;
  const int nt = p.N / bn_out;
  const int tm = BM * cg;
  int hint = p.grouped ? num_sms : ((p.M + tm - 1) / tm) * nt * ks;
  if (swap)
    return epi == EPI_SWIGLU ? launch_impl<256, EPI_SWIGLU, 2, true>(ma, mb, q, hint, num_sms, st)
                             : launch_impl<256, EPI_MERGE_MLP, 2, true>(ma, mb, q, hint, num_sms, st);
#define ZAYA_GEMM_CASE(BNV, EPIV)                                                  \
  if (bn == BNV && epi == EPIV)                                                    \
    return cg == 2 ? launch_impl<BNV, EPIV, 2>(ma, mb, p, hint, num_sms, st)       \
                   : launch_impl<BNV, EPIV, 1>(ma, mb, p, hint, num_sms, st);
  ZAYA_GEMM_CASE(256, EPI_STORE_BF16)
  ZAYA_GEMM_CASE(128, EPI_STORE_BF16)
  ZAYA_GEMM_CASE(64, EPI_STORE_BF16)
  ZAYA_GEMM_CASE(256, EPI_MERGE_ATTN)
  ZAYA_GEMM_CASE(128, EPI_MERGE_ATTN)
  ZAYA_GEMM_CASE(64, EPI_MERGE_ATTN)
  ZAYA_GEMM_CASE(128, EPI_ROUTER_DOWN)
  ZAYA_GEMM_CASE(64, EPI_ROUTER_DOWN)
  ZAYA_GEMM_CASE(32, EPI_ROUTER_DOWN)
  ZAYA_GEMM_CASE(256, EPI_STORE_F32)
  ZAYA_GEMM_CASE(128, EPI_STORE_F32)
  ZAYA_GEMM_CASE(64, EPI_STORE_F32)
  ZAYA_GEMM_CASE(32, EPI_STORE_F32)
  ZAYA_GEMM_CASE(32 * 8, EPI_SWIGLU)
  ZAYA_GEMM_CASE(256, EPI_MERGE_MLP)
  ZAYA_GEMM_CASE(128, EPI_MERGE_MLP)
  ZAYA_GEMM_CASE(64, EPI_MERGE_MLP)
#undef ZAYA_GEMM_CASE
  return ZAYA_ERR_UNSUPPORTED;
}

}  // namespace zaya
