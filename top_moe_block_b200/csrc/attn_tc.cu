// Sliding-window causal GQA attention, prefill, on the 5th-generation tensor
// cores (tcgen05 + TMEM).
//
// softmax(q k^T * scale + mask) v for every query head h with kv head
// h / (n_q / n_kv); key j is visible to query i iff 0 <= i - j < window and
// key j is not padding (nnterp "zaya" page: grouped-query eager softmax
// attention).  A query with no visible key outputs 0.
//
// CTA = 128 queries of one query head, 7 warps, two CTAs per SM (256 TMEM
// columns and ~98 KB of shared memory each), so that one CTA's pipeline fill
// and drain (Q load, first S, the O readout or partial write) overlap the
// other's steady state (measured 72 us against 77 us for one CTA of two heads
// per SM at S = 4096):
//   warp 0     TMA: the head's Q tile once, then K tiles of 64 keys into a
//              2-slot ring (128-byte swizzle, 64-wide d atoms);
//   warp 6     TMA: V tiles into their own 2-slot ring.  K and V have a
//              thread each, so a K tile is requested as soon as its slot is
//              free (S(j) done) rather than behind the previous V tile, whose
//              slot frees only after P V (measured: the softmax waited ~1100
//              cycles per tile for S with one thread loading both);
//   warp 1     one thread issues tcgen05.mma: S(j) = Q K^T into one of two S
//              buffers in tensor memory; once the softmax has written P(j)
//              over it, O += P V with P read straight from tensor memory (A
//              operand in TMEM) and V from shared memory as an MN-major
//              operand, then, once K(j+2) has landed, S(j+2) into the same
//              buffer: S runs two tiles ahead of the softmax, and P V never
//              waits for a K tile;
//   warps 2-5  softmax, one thread per query row (its TMEM lane): row max
//              and sum are thread-local; P goes back into the S columns as
//              bf16 pairs (tcgen05.st).  The running max is only moved (and O
//              rescaled in TMEM) when it grows by more than 2^8, which keeps
//              P <= 256 and the result exact.
// The code is written for kHPC query heads per CTA (sharing the K / V tiles);
// kHPC = 2 with one CTA per SM measured slower.
// Shared memory carries only Q, K and V (P never leaves tensor memory): a
// version with P staged in shared memory was measured to be limited by
// shared-memory bandwidth, and one with a single S buffer per head by the
// serial S -> softmax -> PV -> S chain.
// Only key tiles that intersect the window are visited; per-element masks
// only on tiles that straddle the diagonal, the window edge, the sequence
// end or a padding mask.
// Balance: causal rows differ in length (row tile i of a short sequence sees
// i+1 key tiles), so when the longest row tile holds more key tiles than a
// CTA slot's share of the whole launch (two slots per SM), row tiles are cut
// into key chunks of at most two thirds of that share.  The host lists the
// (row tile, chunk, head, sequence) items longest first; a chunk writes its unnormalised O with its
// running max and sum (fp32), and the last chunk of a row tile to finish
// (a per-row-tile counter) merges all chunks in chunk order:
// O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c, M = max_c m_c.
#include <algorithm>
#include <vector>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace zaya {

namespace {

constexpr int kQT = 128;  // queries per CTA
constexpr int kKT = 64;   // keys per tile
constexpr int kHPC = 1;   // query heads per CTA (sharing one kv head)
constexpr int kRing = 2;  // K ring depth (S runs two tiles ahead)
constexpr int kRingV = 2; // V ring depth
constexpr float kRescaleLog2 = 8.0f;
constexpr int kMaxItems = 1024;  // split-plan items carried in the kernel parameters (16 KB)
constexpr int kPlanSms = 296;    // the CTA slots the split plan balances over (148 SMs x 2)
constexpr int kMinChunk = 4;     // fewest key tiles in a chunk
constexpr int kVWarp = 2 + 4 * kHPC;            // the V loader
constexpr int kThreads = 32 * (kVWarp + 1);     // producer, MMA, softmax warpgroups, V loader

struct AttnItems {
  int n_items;   // 0: grid (row tiles, head groups of kHPC, sequences), no row tile split
  float* po;     // partial O, per slot [kHPC][d][kQT] fp32 (row index fastest)
  float* pml;    // per slot [kHPC][2][kQT] fp32: running max (log2 units), running sum
  int* ctr;      // per split (row tile, head group, sequence): chunks finished
  uint4 it[kMaxItems];   // {rt | c << 16 | nc << 24, b | hp << 16, first slot of the group, counter}
};

// Key tiles of row tile rt (the same arithmetic as the kernel's).
inline int host_row_tiles(int rt, int S, int window) {
  const int m0 = rt * kQT;
  const int lo = std::max(0, m0 - window + 1);
  const int n_begin = (lo / kKT) * kKT;
  const int n_end = std::min(S, m0 + kQT);
  return (n_end - n_begin + kKT - 1) / kKT;
}

// The split plan: fills `items` (when non-null) and the slot / counter counts.
// Returns false when no row tile is split.
bool plan_split(int B, int S, int window, int n_hp, AttnItems* items, int* n_slots, int* n_ctr) {
  *n_slots = 0;
  *n_ctr = 0;
  if (items) items->n_items = 0;
  const int n_rt = (S + kQT - 1) / kQT;
  long total = 0;
  int maxnt = 0;
  for (int rt = 0; rt < n_rt; ++rt) {
    const int nt = host_row_tiles(rt, S, window);
    total += nt;
    maxnt = std::max(maxnt, nt);
  }
  total *= (long)B * n_hp;
  const double share = (double)total / kPlanSms;
  if (maxnt <= share) return false;
  // chunks of about two thirds of an SM's share: the in-order CTA dispatch
  // then pairs the first round's long items with the later rounds' short
  // ones.  Each item costs a pipeline fill and drain (Q load, first S, the O
  // readout or partial write), so much shorter chunks lose more than the
  // finer balance gains (measured at S = 4096: share/1.5 beat share, share/2
  // and share/3).
  for (int L = std::max(kMinChunk, (int)(share / 1.5 + 0.999)); L < maxnt; L *= 2) {
    long n_items = 0, slots = 0, ctrs = 0;
    bool fits = true;
    for (int rt = 0; rt < n_rt && fits; ++rt) {
      const int nc = (host_row_tiles(rt, S, window) + L - 1) / L;
      if (nc > 255) fits = false;
      n_items += (long)nc * n_hp * B;
      if (nc > 1) {
        slots += (long)nc * n_hp * B;
        ctrs += (long)n_hp * B;
      }
    }
    if (!fits || n_items > kMaxItems || B > 0xffff || n_hp > 0xffff || n_rt > 0xffff) continue;
    *n_slots = (int)slots;
    *n_ctr = (int)ctrs;
    if (items) {
      struct It { int size; uint4 v; };
      std::vector<It> v;
      int slot = 0, ctr = 0;
      for (int rt = n_rt - 1; rt >= 0; --rt) {
        const int nt = host_row_tiles(rt, S, window);
        const int nc = (nt + L - 1) / L;
        for (int hp = 0; hp < n_hp; ++hp)
          for (int b = 0; b < B; ++b) {
            const int s0 = slot, c0 = ctr;
            if (nc > 1) {
              slot += nc;
              ++ctr;
            }
            for (int c = 0; c < nc; ++c) {
              const int size = (c + 1) * nt / nc - c * nt / nc;
              v.push_back({size, make_uint4((uint32_t)rt | ((uint32_t)c << 16) | ((uint32_t)nc << 24),
                                            (uint32_t)b | ((uint32_t)hp << 16), (uint32_t)s0, (uint32_t)c0)});
            }
          }
      }
      std::stable_sort(v.begin(), v.end(), [](const It& a, const It& b) { return a.size > b.size; });
      items->n_items = (int)v.size();
      for (size_t i = 0; i < v.size(); ++i) items->it[i] = v[i].v;
    }
    return true;
  }
  return false;
}

size_t slot_bytes(int d) { return (size_t)kHPC * d * kQT * 4 + (size_t)kHPC * 2 * kQT * 4; }

template <int D>
struct AttnTc {
  static constexpr int SUB = D / 64;               // 64-wide swizzle atoms along d
  static constexpr int Q_ATOM = kQT * 128;         // [128 rows][64] bf16 atom: 16 KB
  static constexpr int KV_ATOM = kKT * 128;        // [64 keys][64] bf16 atom: 8 KB
  static constexpr int Q_BYTES = SUB * Q_ATOM;     // one head's Q tile
  static constexpr int KV_BYTES = SUB * KV_ATOM;   // one K (or V) tile
  static constexpr int SMEM_USED = 1024 + kHPC * Q_BYTES + (kRing + kRingV) * KV_BYTES + 512;
  static constexpr int SMEM = SMEM_USED;           // two CTAs per SM
  static_assert(2 * (SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
  // per head: S0 / P0 [0, 64), S1 / P1 [64, 128), O [128, 128 + D); two CTAs share the 512 columns
  static constexpr uint32_t TMEM_COLS = kHPC * 256;
  static constexpr uint32_t HEAD_COLS = 256;
  static constexpr uint32_t O_COL = 2 * kKT;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, kKT);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32_bmn(128, D);
  static_assert(kHPC * (2 * kKT + D) <= 256, "tensor memory: two CTAs per SM");
};

// 2^x on the special-function unit (inputs <= 0 here; results below 2^-126
// flush to zero, which a softmax weight can drop).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool key_visible(int q, int key, int window, int S, const int* mask) {
  return key <= q && q - key < window && key < S && (!mask || mask[key] != 0);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p,
                   const __grid_constant__ AttnItems items, int* status) {
  using C = AttnTc<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                           // [kHPC] Q tiles
  uint8_t* sK = sQ + kHPC * C::Q_BYTES;         // [kRing] K tiles
  uint8_t* sV = sK + kRing * C::KV_BYTES;       // [kRingV] V tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kRingV * C::KV_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                  // [kRing]
  uint64_t* k_empty = k_full + kRing;           // [kRing]
  uint64_t* v_full = k_empty + kRing;           // [kRingV]
  uint64_t* v_empty = v_full + kRingV;          // [kRingV]
  uint64_t* s_full = v_empty + kRingV;          // [kHPC][2]: S(j) of the head is in S buffer j & 1
  uint64_t* p_full = s_full + 2 * kHPC;         // [kHPC][2]: P(j) is in TMEM over S(j)
  uint64_t* pv_done = p_full + 2 * kHPC;        // [kHPC]: O += P(j) V(j) complete
  uint64_t* o_ready = pv_done + kHPC;           // the MMA thread's last commit: every MMA of the CTA is done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_ready + 1);
  int* s_last = reinterpret_cast<int*>(tmem_slot + 1);

  // this CTA's item: a row tile of its kHPC heads, or one key chunk of it
  int qb, hp, b, chunk = 0, n_chunks = 1, slot0 = 0, ctr = 0;
  if (items.n_items) {
    const uint4 it = items.it[blockIdx.x];
    qb = (int)(it.x & 0xffff);
    chunk = (int)((it.x >> 16) & 0xff);
    n_chunks = (int)(it.x >> 24);
    b = (int)(it.y & 0xffff);
    hp = (int)(it.y >> 16);
    slot0 = (int)it.z;
    ctr = (int)it.w;
  } else {
    qb = gridDim.x - 1 - blockIdx.x;   // heaviest (latest) query tiles first
    hp = blockIdx.y;
    b = blockIdx.z;
  }
  const int h0 = hp * kHPC;
  const int g = h0 / (p.n_q / p.n_kv);
  const int m0 = qb * kQT;
  const int S = p.S;
  const int lo = max(0, m0 - p.window + 1);
  const int n_begin = (lo / kKT) * kKT;
  const int n_end = min(S, m0 + kQT);
  const int n_row_tiles = (n_end - n_begin + kKT - 1) / kKT;
  const int t_begin = chunk * n_row_tiles / n_chunks;
  const int n_tiles = (chunk + 1) * n_row_tiles / n_chunks - t_begin;   // key tiles of this item
  const int warp = warp_id(), lane = lane_id();

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kRingV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2 * kHPC; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
    }
    for (int i = 0; i < kHPC; ++i) mbar_init(&pv_done[i], 1);
    mbar_init(o_ready, 1);
    fence_barrier_init();
    fence_proxy_async();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_begin();   // the prologue above overlaps the previous kernel; global memory only from here
  // A fault already recorded (an earlier wait ran out) means the launch chain
  // has failed: no work.  Each role reads the word itself; roles that read
  // differently meet in waits that give up on the recorded fault.
  const WaitCtx wc = wait_ctx(status);
  const int n_work = wc.skip ? 0 : n_tiles;

  if (warp == 0) {
    // ---------------- TMA producer: the heads' Q once, then K(j) into its ring
    if (elect_one() && !wc.skip) {
      const int kv_row = (b * p.n_kv + g) * p.cap + n_begin + t_begin * kKT;
      mbar_arrive_expect_tx(q_full, kHPC * C::Q_BYTES);
#pragma unroll
      for (int x = 0; x < kHPC; ++x) {
        const int q_row = (b * p.n_q + h0 + x) * S + m0;
#pragma unroll
        for (int s = 0; s < C::SUB; ++s)
          tma_load_2d(sQ + x * C::Q_BYTES + s * C::Q_ATOM, &tmQ, q_full, s * 64, q_row);
      }
      int nk = 0;   // K tiles whose copies were started
      for (int j = 0; j < n_tiles; ++j) {
        const int slot = j % kRing;
        const uint32_t par = ((j / kRing) & 1) ^ 1u;
        if (!mbar_wait(&k_empty[slot], par, wc)) break;
        mbar_arrive_expect_tx(&k_full[slot], C::KV_BYTES);
#pragma unroll
        for (int s = 0; s < C::SUB; ++s)
          tma_load_2d(sK + slot * C::KV_BYTES + s * C::KV_ATOM, &tmK, &k_full[slot], s * 64, kv_row + j * kKT);
        ++nk;
      }
      // every copy started must land before the CTA may exit: the last phase
      // armed on each slot (tile j uses phase j / ring of slot j % ring)
      mbar_drain(q_full, 0, status);
      for (int j = (nk > kRing ? nk - kRing : 0); j < nk; ++j) mbar_drain(&k_full[j % kRing], (j / kRing) & 1, status);
    }
  } else if (warp == kVWarp) {
    // ---------------- TMA producer: V(j) into its ring
    if (elect_one() && !wc.skip) {
      const int kv_row = (b * p.n_kv + g) * p.cap + n_begin + t_begin * kKT;
      int nv = 0;   // V tiles whose copies were started
      for (int j = 0; j < n_tiles; ++j) {
        const int vslot = j % kRingV;
        if (!mbar_wait(&v_empty[vslot], ((j / kRingV) & 1) ^ 1u, wc)) break;
        mbar_arrive_expect_tx(&v_full[vslot], C::KV_BYTES);
#pragma unroll
        for (int s = 0; s < C::SUB; ++s)
          tma_load_2d(sV + vslot * C::KV_BYTES + s * C::KV_ATOM, &tmV, &v_full[vslot], s * 64, kv_row + j * kKT);
        ++nv;
      }
      for (int j = (nv > kRingV ? nv - kRingV : 0); j < nv; ++j)
        mbar_drain(&v_full[j % kRingV], (j / kRingV) & 1, status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer.  Per head: S(j) into S buffer j & 1; the
    // softmax writes P(j) over it; O += P(j) V(j) with P read from tensor
    // memory; then S(j+2) into the same buffer (the tensor pipe runs one
    // thread's MMAs in issue order, so S(j+2) is written after P(j) is read).
    // S runs two tiles ahead of the softmax (with kHPC > 1 the heads alternate).
    if (elect_one()) {
      bool ok = n_work > 0 && mbar_wait(q_full, 0, wc);
      auto issue_qk = [&](int x, int j) {
        const uint32_t ka = smem_u32(sK + (j % kRing) * C::KV_BYTES);
        const uint32_t qa = smem_u32(sQ + x * C::Q_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          tc_mma_bf16(tmem_base + x * C::HEAD_COLS + (j & 1) * kKT,
                      smem_desc_sw128(qa + (kk >> 2) * C::Q_ATOM + koff, 16, 1024),
                      smem_desc_sw128(ka + (kk >> 2) * C::KV_ATOM + koff, 16, 1024), C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[x * 2 + (j & 1)]);
      };
      for (int j = 0; ok && j < 2 && j < n_tiles; ++j) {   // S(0), S(1)
        ok = mbar_wait(&k_full[j], 0, wc);
        if (!ok) break;
        tc_fence_after();
        for (int x = 0; x < kHPC; ++x) issue_qk(x, j);
        tc_commit(&k_empty[j]);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int vslot = j % kRingV, nslot = (j + 2) % kRing;
        const bool more = j + 2 < n_tiles;
        if (!mbar_wait(&v_full[vslot], (j / kRingV) & 1, wc)) break;
        const uint32_t va = smem_u32(sV + vslot * C::KV_BYTES);
        for (int x = 0; ok && x < kHPC; ++x) {
          if (!mbar_wait(&p_full[x * 2 + (j & 1)], (j >> 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t pa = tmem_base + x * C::HEAD_COLS + (j & 1) * kKT;   // P(j): bf16 pairs over S(j)
#pragma unroll
          for (int kk = 0; kk < kKT / 16; ++kk)
            tc_mma_bf16_ts(tmem_base + x * C::HEAD_COLS + C::O_COL, pa + kk * 8,
                           smem_desc_sw128(va + kk * 2048, C::KV_ATOM, 1024), C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&pv_done[x]);
        }
        if (!ok) break;
        tc_commit(&v_empty[vslot]);
        if (more) {   // S(j+2) once K(j+2) has landed, after P V(j) in the pipe's order
          if (!mbar_wait(&k_full[nslot], ((j + 2) / kRing) & 1, wc)) break;
          tc_fence_after();
          for (int x = 0; x < kHPC; ++x) issue_qk(x, j + 2);
          tc_commit(&k_empty[nslot]);
        }
      }
      // the last commit, issued on every path: it arrives once every MMA above
      // has completed -- O is final and the tensor memory may be freed
      tc_commit(o_ready);
      mbar_drain(o_ready, 0, status);
    }
  } else {
    // ---------------- softmax: warpgroup x handles head h0 + x, one thread per query row
    const int x = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int q = m0 + row;
    const uint32_t tl = tmem_base + x * C::HEAD_COLS + ((uint32_t)(quarter * 32) << 16);
    const int* mask = p.mask ? p.mask + (size_t)b * S : nullptr;
    const float sl2 = p.scale * 1.4426950408889634f;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_work; ++j) {
      // every wait that guards a .sync.aligned TMEM access is made warp-uniform
      const int buf = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[x * 2 + buf], (j >> 1) & 1, wc))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int key0 = n_begin + (t_begin + j) * kKT;
      const bool full_vis = !mask && key0 + kKT - 1 <= m0 && (m0 + kQT - 1 - key0) < p.window && key0 + kKT <= S;
      uint32_t r[kKT];
#pragma unroll
      for (int c = 0; c < kKT / 32; ++c)
        tmem_ld32(tl + buf * kKT + c * 32, *reinterpret_cast<uint32_t(*)[32]>(r + c * 32));
      tmem_ld_wait();
      float* v = reinterpret_cast<float*>(r);
      if (full_vis) {
#pragma unroll
        for (int i = 0; i < kKT; ++i) v[i] = __uint_as_float(r[i]) * sl2;
      } else {
#pragma unroll
        for (int i = 0; i < kKT; ++i) {
          const float xv = __uint_as_float(r[i]) * sl2;
          v[i] = key_visible(q, key0 + i, p.window, S, mask) ? xv : -INFINITY;
        }
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four independent chains
#pragma unroll
      for (int i = 0; i < kKT; ++i) mx[i & 3] = fmaxf(mx[i & 3], v[i]);
      const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      const float m_new = fmaxf(m_used, tmax);
      // Move the running max when it grew by more than 2^8 -- for the whole warp
      // at once, since the O rescale below is a warp-wide TMEM access.  Each
      // lane scales its own row by exp2(m_used - m_new) <= 1, so the result is
      // exact whichever lanes asked.
      if (__any_sync(0xffffffffu, m_new > m_used + kRescaleLog2)) {
        const bool finite_new = m_new != -INFINITY;
        const float f = (m_used == -INFINITY || !finite_new) ? 1.f : exp2f(m_used - m_new);
        if (j > 0 && __any_sync(0xffffffffu, m_used != -INFINITY)) {
          // O holds tiles < j: wait for PV(j-1), then scale O in TMEM
          // S(j) was committed after PV(j-2), so pv_done is at most one phase behind
          // PV(j-1) here and its parity names that phase unambiguously
          if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[x], (j - 1) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tl + C::O_COL + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(tl + C::O_COL + c * 32, o);
          }
          tmem_st_wait();
        }
        l *= f;
        if (finite_new) m_used = m_new;
      }
      const float base = (m_used == -INFINITY) ? 0.f : m_used;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      // P = 2^(v - base) as bf16 pairs, written over the first kKT/2 columns of S(j)
#pragma unroll
      for (int c = 0; c < kKT / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2_approx(v[c * 32 + i] - base), p1 = ex2_approx(v[c * 32 + i + 1] - base);
          ls[(i >> 1) & 3] += p0 + p1;
          pk[i >> 1] = pack_bf2(p0, p1);
        }
        tmem_st16(tl + buf * kKT + c * 16, pk);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[x * 2 + buf]);
    }
    // O is final once the MMA thread's last commit has arrived (a single-use
    // barrier: pv_done could still be two phases short of PV(n-1) here, when
    // PV(n-2) has not completed, which its parity cannot tell apart)
    const bool have = ok && n_work > 0 && __all_sync(0xffffffffu, mbar_wait(o_ready, 0, wc));
    const int ld = p.n_q * D;
    auto* out = static_cast<__nv_bfloat16*>(p.out) + ((size_t)b * S + q) * ld + (h0 + x) * D;
    // this row's 32 output columns [c, c + 32), scaled, as bf16
    auto store32 = [&](int c, const float* v, float sc) {
      if (q >= S) return;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint4 vv;
        vv.x = pack_bf2(v[8 * u + 0] * sc, v[8 * u + 1] * sc);
        vv.y = pack_bf2(v[8 * u + 2] * sc, v[8 * u + 3] * sc);
        vv.z = pack_bf2(v[8 * u + 4] * sc, v[8 * u + 5] * sc);
        vv.w = pack_bf2(v[8 * u + 6] * sc, v[8 * u + 7] * sc);
        reinterpret_cast<uint4*>(out + c)[u] = vv;
      }
    };
    if (n_chunks == 1) {
      if (have) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tl + C::O_COL + c * 32, o);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]);
          store32(c * 32, v, inv);
        }
      }
    } else {
      // unnormalised partial of this key chunk: O transposed (row fastest, so a
      // warp's stores are contiguous), running max and sum
      float* po = items.po + ((size_t)(slot0 + chunk) * kHPC + x) * D * kQT;
      float* pml = items.pml + ((size_t)(slot0 + chunk) * kHPC + x) * 2 * kQT;
      if (have) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tl + C::O_COL + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) po[(size_t)(c * 32 + i) * kQT + row] = __uint_as_float(o[i]);
        }
        pml[row] = m_used;
        pml[kQT + row] = l;
      }
      __threadfence();
      named_barrier_sync(1, 32 * 4 * kHPC);
      if (warp == 2 && lane == 0) *s_last = (atomicAdd(items.ctr + ctr, 1) == n_chunks - 1);
      named_barrier_sync(1, 32 * 4 * kHPC);
      if (*s_last) {   // every chunk of this row tile is written: merge in chunk order
        __threadfence();
        auto ml = [&](int cc, int which) {
          return __ldcg(items.pml + ((size_t)(slot0 + cc) * kHPC + x) * 2 * kQT + which * kQT + row);
        };
        float M = -INFINITY;
        for (int cc = 0; cc < n_chunks; ++cc) M = fmaxf(M, ml(cc, 0));
        float Ls = 0.f;
        for (int cc = 0; cc < n_chunks; ++cc) {
          const float mc = ml(cc, 0);
          if (mc != -INFINITY) Ls += exp2f(mc - M) * ml(cc, 1);
        }
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float acc[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = 0.f;
          for (int cc = 0; cc < n_chunks; ++cc) {
            const float mc = ml(cc, 0);
            if (mc == -INFINITY) continue;
            const float w = exp2f(mc - M);
            const float* pc = items.po + ((size_t)(slot0 + cc) * kHPC + x) * D * kQT + (size_t)c * 32 * kQT + row;
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = fmaf(w, __ldcg(pc + (size_t)i * kQT), acc[i]);
          }
          store32(c * 32, acc, inv);
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace

size_t attn_prefill_ws_bytes(int B, int S, int window, int n_q, int n_kv, int d) {
  if (B <= 0 || S <= 0 || n_q % kHPC) return 0;
  int n_slots = 0, n_ctr = 0;
  if (!plan_split(B, S, window, n_q / kHPC, nullptr, &n_slots, &n_ctr)) return 0;
  return (size_t)n_slots * slot_bytes(d) + (size_t)n_ctr * 4;
}

int attn_prefill_ctr(int B, int S, int window, int n_q, int d, size_t* byte_off) {
  *byte_off = 0;
  if (B <= 0 || S <= 0 || n_q % kHPC) return 0;
  int n_slots = 0, n_ctr = 0;
  if (!plan_split(B, S, window, n_q / kHPC, nullptr, &n_slots, &n_ctr)) return 0;
  *byte_off = (size_t)n_slots * slot_bytes(d);
  return n_ctr;
}

int launch_attn_prefill_tc(const AttnParams& p, int* status, cudaStream_t st) {
  if (p.B <= 0 || p.S <= 0) return ZAYA_OK;
  if (p.d != 128 && p.d != 64) return ZAYA_ERR_UNSUPPORTED;
  if (p.n_q % kHPC || (p.n_q / p.n_kv) % kHPC) return ZAYA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  int rc = make_tmap_bf16(&mq, p.q, (uint64_t)p.B * p.n_q * p.S, (uint64_t)p.d, 128);
  if (!rc) rc = make_tmap_bf16(&mk, p.k_cache, (uint64_t)p.B * p.n_kv * p.cap, (uint64_t)p.d, kKT);
  if (!rc) rc = make_tmap_bf16(&mv, p.v_cache, (uint64_t)p.B * p.n_kv * p.cap, (uint64_t)p.d, kKT);
  if (rc) return rc;
  AttnItems items;   // the kernel's item parameter (8 KB, copied at launch)
  int n_slots = 0, n_ctr = 0;
  dim3 grid((p.S + kQT - 1) / kQT, p.n_q / kHPC, p.B);
  if (plan_split(p.B, p.S, p.window, p.n_q / kHPC, &items, &n_slots, &n_ctr)) {
    const size_t need = (size_t)n_slots * slot_bytes(p.d) + (size_t)n_ctr * 4;
    if (!p.part || p.part_bytes < need) return ZAYA_ERR_WORKSPACE;
    items.po = static_cast<float*>(p.part);
    items.pml = items.po + (size_t)n_slots * kHPC * p.d * kQT;
    items.ctr = reinterpret_cast<int*>(items.pml + (size_t)n_slots * kHPC * 2 * kQT);
    if (!p.ctr_cleared && cudaMemsetAsync(items.ctr, 0, (size_t)n_ctr * 4, st) != cudaSuccess) return ZAYA_ERR_CUDA;
    grid = dim3(items.n_items, 1, 1);
  } else {
    items.n_items = 0;
    items.po = items.pml = nullptr;
    items.ctr = nullptr;
  }
  if (p.d == 128) {
    auto kern = attn_tc_kernel<128>;
    static bool set = false;
    if (!set) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnTc<128>::SMEM);
      set = true;
    }
    launch_k(kern, grid, dim3(kThreads), AttnTc<128>::SMEM, st, nullptr, 0, mq, mk, mv, p, items, status);
  } else {
    auto kern = attn_tc_kernel<64>;
    static bool set = false;
    if (!set) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnTc<64>::SMEM);
      set = true;
    }
    launch_k(kern, grid, dim3(kThreads), AttnTc<64>::SMEM, st, nullptr, 0, mq, mk, mv, p, items, status);
  }
  return cudaGetLastError() == cudaSuccess ? ZAYA_OK : ZAYA_ERR_CUDA;
}

}  // namespace zaya
