// Internal launchers of the ZAYA1 block kernels (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace zaya {

// ------------------------------------------------------------------ GEMM
enum EpiKind {
  EPI_STORE_BF16 = 0,   // out[m, n] = bf16(acc)
  EPI_MERGE_ATTN = 1,   // o_proj + merge 1, stream updated in place
  EPI_ROUTER_DOWN = 2,  // out[m, n] = acc + bias[n] (+ prev[m, n] * scale[n]) in fp32
  EPI_SWIGLU = 3,       // grouped: act = bf16(silu(gate) * up)
  EPI_MERGE_MLP = 4,    // grouped: expert down + weight + merge 2, scattered to token rows
  EPI_STORE_F32 = 5     // out[split][m, n] = acc (fp32 partial sums of a split-K product)
};

struct GemmParams {
  int M, N, K;               // C[M, N] = A[M, K] * B[N, K]^T (N = output columns)
  int k_splits;              // dense STORE_F32 only: K split into this many slabs (0 or 1: none)
  int grouped;               // expert-grouped A rows / B row blocks
  const int* group_off;      // [E+1] first A row of each expert (grouped)
  const int* mt_start;       // [E+1] prefix of per-expert tile counts (grouped; 128-row tiles, 256 with pair)
  int pair;                  // 1: CTA-pair kernel (cta_group::2), 256-row tiles; bn 128 or 256
  int n_groups;              // E
  int b_rows_per_group;      // rows of B per expert (2I or H)
  int* status;
  void* out;                 // STORE_BF16 / SWIGLU: bf16 [rows, ldo]; ROUTER_DOWN: fp32 [M, ldo];
                             // STORE_F32: fp32 [k_splits, M, ldo]
  int ldo;
  float* stream;             // MERGE_*: fp32 [tokens, N]
  const float* merge;        // MERGE_*: fp32 [4, N] hb, hs, rb, rs
  const float* bias;         // ROUTER_DOWN [N]
  const float* prev;         // ROUTER_DOWN [M, N] or null
  const float* prev_scale;   // ROUTER_DOWN [N]
  const int* perm;           // MERGE_MLP: permuted row -> token
  const float* row_w;        // MERGE_MLP: per-token expert weight
  void* tap_bf16;            // MERGE_*: optional bf16 [tokens, N] contribution tap
  float* tap_f32;            // MERGE_ATTN: optional fp32 [tokens, N] layer_mid tap
  int tok_box;               // set by launch_gemm: swapped tiles' token box rows (16)
  int fp8;                   // grouped experts: A rows and B weights are E4M3 bytes (tcgen05 kind::f8f6f4)
  const float* w_scale;      // fp8: [E, b_rows_per_group] fp32 per-row weight scales
  const float* act_scale;    // fp8: [E, 2] static input scales (gate/up input, down input)
};

// Encodes a 2-D bf16 tensor map (rows x cols, row-major) with a box of
// box_rows x 64 and the 128-byte swizzle.  Returns 0 on success.
int make_tmap_bf16(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);

// Launches the tcgen05 GEMM; bn = 64, 128 or 256 (SWIGLU: 128 output
// columns per tile, 256 MMA columns).  A and B maps are built inside.
int launch_gemm(int epi, int bn, const void* A, int a_rows, const void* B, int b_rows, const GemmParams& p,
                int num_sms, cudaStream_t st);

// Router down-projection plan for M rows and R outputs over K inputs.
// 0: one pass over K whose epilogue adds the bias and the carried state and
// writes the router state itself, chosen when 64-column tiles alone give 96 or
// more CTAs.  Otherwise the number of K slabs (a power of two, at most 8 and
// K/64) of fp32 partial sums that the router kernel adds in slab order: enough
// 128-row x slab tiles to fill the GPU while the slabs stay small.
// Deterministic in (M, R, K).
inline int router_down_splits(int M, int R, int K) {
  const int mt = (M + 127) / 128;
  if (R % 64 == 0 && mt * (R / 64) >= 96) return 0;
  int ks = 1;
  while (ks * 2 <= 8 && ks * 2 <= K / 64 && mt * ks * 2 <= 148) ks *= 2;
  return ks;
}

// ------------------------------------------------------------------ norms
// out[m] = bf16(w * xb * rsqrt(mean(xb^2) + eps)), xb = bf16(x[m * row_mul +
// row_add]); extra rows [M, M+n_copy) of out are a copy of copy_src (decode:
// prev_hs, whose projection gives the delayed values).
int launch_rmsnorm(const float* x, int row_mul, int row_add, const void* w, void* out, void* tap, int M, int H,
                   float eps, const void* copy_src, int n_copy, cudaStream_t st);
int launch_embed(const int* ids, const void* table, float* stream, int M, int H, int vocab, float mult,
                 float shift, int* status, cudaStream_t st);

// ------------------------------------------------------------------ CCA attention input
struct CcaParams {
  const void* qkv;        // bf16 [rows, n_qkv]
  int n_qkv;
  const float* conv_w;    // [C, 3]
  const float* conv_b;    // [C]
  const float* k_temp;    // [n_kv]
  const int* mask;        // prefill [B, S] or null
  void* q_out;            // bf16 [B, n_q, S, d]
  void* tap_q;            // optional copy of q_out
  void* k_cache;
  void* v_cache;
  int cache_cap;
  int* cache_len;         // [B]
  void* conv_state;       // bf16 [B, C, 2]
  void* prev_hs;          // bf16 [B, H]
  const void* a_in;       // bf16 [rows, H] (prev_hs source)
  int B, S, H, n_q, n_kv, d, rot;
  int cca_res, v_delayed;
  float theta, eps;
  int decode;             // 1: one token per sequence, history from conv_state
  int ring;               // decode: 1 = the caches are window rings (position p at slot p % cache_cap)
  int fp8;                // decode: 1 = the caches hold E4M3 bytes
  int* status;
  int* zero_words;        // prefill: words CTA 0 clears for the next kernel (attention's merge counters), or null
  int n_zero_words;
  const float* conv_y;    // fp32 [rows, C]: the two-stage conv's output (used instead of the width-3 conv), or null
  float inv_freq[64];     // RoPE inverse frequencies theta^(-2i/rot), i < rot/2 (fp32)
};
int launch_cca(const CcaParams& p, cudaStream_t st);
// Prefill into a window ring or an fp8 cache: positions max(0, S - cap) ..
// S-1 of the linear bf16 K / V ([B, n_kv, S, d]) into the caches ([B, n_kv,
// cap, d]) at slot p (ring: p % cap), as bf16 or (fp8) E4M3 bytes.
int launch_cache_store(const void* k_lin, const void* v_lin, void* k_cache, void* v_cache, int B, int n_kv, int S,
                       int cap, int d, int ring, int fp8, int* status, cudaStream_t st);

// The two-stage conv_qk's grouped stage (with its depthwise stage fused in):
// y fp32 [rows, C], one group per q / k head.
struct ConvGroupedParams {
  const void* qkv;        // bf16 [rows, ld]: the pre-conv q||k projection in columns [0, C)
  int ld;
  const float* dw;        // [C, 2] depthwise taps (t-1, t)
  const float* db;        // [C]
  const float* gw;        // [C, D, 2] grouped taps (Conv1d layout [out, in / groups, k])
  const float* gb;        // [C]
  const int* mask;        // prefill [B, S] or null
  const void* conv_state; // decode: bf16 [rows, C, 2] (u at t-2, t-1)
  float* y;               // [rows, C]
  int rows, S, C, decode;
};
int launch_conv_grouped(const ConvGroupedParams& p, int groups, int d, int num_sms, cudaStream_t st);

// ------------------------------------------------------------------ attention
struct AttnParams {
  const void* q;          // bf16 [B, n_q, S, d]
  const void* k_cache;    // bf16 [B, n_kv, cap, d]
  const void* v_cache;
  const int* mask;        // [B, S] or null
  void* out;              // bf16 premix [B*S, n_q*d]
  int B, S, cap, n_q, n_kv, d, window;
  float scale;
  void* part;             // split-KV partials + merge counters (attn_prefill_ws_bytes)
  size_t part_bytes;
  int ctr_cleared;        // 1: the merge counters (attn_prefill_ctr) were cleared by the previous kernel
};
// The merge counters inside `part` for these sizes: returns their count (0
// without a split) and their byte offset; they must be zero at launch.
int attn_prefill_ctr(int B, int S, int window, int n_q, int d, size_t* byte_off);
// Workspace bytes of the split-KV plan for these sizes (0 when no row tile is split).
size_t attn_prefill_ws_bytes(int B, int S, int window, int n_q, int n_kv, int d);
int launch_attn_prefill_tc(const AttnParams& p, int* status, cudaStream_t st);

struct DecodeAttnParams {
  const void* q;          // bf16 [B, n_q, d]
  const void* k_cache;
  const void* v_cache;
  const int* cache_len;   // [B]: position of the new token (already in the cache)
  void* out;              // bf16 premix [B, n_q*d]
  float* part;            // workspace partials
  int B, cap, n_q, n_kv, d, window, n_chunks;
  int chunk_keys;         // keys per CTA (a multiple of 256)
  int ring;               // 1: position p at slot p % cap
  int fp8;                // 1: the caches hold E4M3 bytes
  float scale;
};
// Key chunks a head's decode attention may use for a window (256 keys per
// chunk, at most 64 chunks; a full-attention block passes a window no cache reaches).
int decode_attn_max_chunks(int window);
// Workspace of the decode attention's partials for up to max_chunks chunks per head.
size_t decode_attn_ws_bytes(int B, int n_q, int d, int max_chunks);
// Key chunks for a span of keys: 256 keys per chunk up to max_chunks, longer chunks beyond it.
void decode_attn_split(int span, int max_chunks, int* n_chunks, int* chunk_keys);
int launch_attn_decode(const DecodeAttnParams& p, cudaStream_t st);

// ------------------------------------------------------------------ router / MoE dispatch
struct RouterParams {
  const float* part;      // [n_splits, M, R] partial sums of m_in . W_down^T (split over K)
  int n_splits;           // 0: r_out already holds the state (bias and carried state added)
  const float* bias;      // [R] down_proj bias
  const float* prev;      // [M, R] previous block's router state, or null (block 0)
  const float* prev_scale;// [R] router_states_scale
  float* r_out;           // [M, R] router state out (= router_state_out)
  const float* norm_w;
  const float* fc1_w; const float* fc1_b;
  const float* fc2_w; const float* fc2_b;
  __nv_bfloat16* wsplit;  // workspace bf16: [2 layers][hi|lo][R][R] (fc1, fc2), then [hi|lo][NP][R] (out_proj, E+1 rows padded to 8)
  const float* out_w;     // [E+1, R]
  const float* balancing; // [E+1]
  const int* mask;        // [M] token validity or null
  float* logits;          // [M, E+1]
  int* cls;               // [M] 0..E (E = skip)
  int* idx;               // optional [M]
  float* w;               // [M]
  float* w_tap;           // optional [M]
  int* class_count;       // [E+1] tokens per class (cleared by the launch, then one atomic add per CTA and class)
  int* lo_any;            // [n_lo_words]: per weight-split block, whether a weight has a nonzero lo part
  int n_lo_words;         // router_split_blocks(R, E)
  int* slot;              // [M]: the token's place among its class's rows (order across CTAs unspecified)
  int* status;            // device status word (a bounded wait that ran out records ZAYA_ERR_TIMEOUT)
  int M, R, E;
  float eps;
};
int launch_router(const RouterParams& p, cudaStream_t st);
// Blocks of the router's weight-split kernel (one lo_any word each).
int router_split_blocks(int R, int E);


// Copies m_in rows of routed tokens into their permuted rows; writes the
// merge-2 output of skipped (and padding) tokens; decode: cache_len += 1.
struct DispatchParams {
  const int* cls;
  const int* class_count; // [E+1] tokens per class (from the router)
  const int* slot;        // [M] place of the token among its class's rows
  int* pos;               // [M] out: permuted row of the token
  int* perm;              // [M] out: token of each permuted row
  int* group_off;         // [E+2] out: first permuted row of each class (written by CTA 0)
  int* mt_start;          // [E+2] out: prefix of per-expert tile counts (tile_rows rows) (CTA 0)
  int tile_rows;
  const void* m_in;       // bf16 [M, H]
  void* x_perm;           // bf16 [M, H]; with in_scale E4M3 bytes of m_in / in_scale[2e]
  const float* in_scale;  // FP8 experts: [E, 2] static input scales, or null
  float* stream;          // [M, H] in: layer_mid; skip rows -> layer_output
  const float* merge_m;   // [4, H]
  void* tap_mlp_out;      // optional bf16 [M, H]
  int* cache_len_inc;     // optional [M] (decode)
  const int* status;      // device status word: a recorded fault makes the kernel do nothing
  int M, H, E;
};
int launch_dispatch(const DispatchParams& p, cudaStream_t st);

int num_sms_current();

}  // namespace zaya
