// C ABI of the ZAYA1 block forward: argument checks, workspace planning and
// the launch sequence of one block (prefill and decode) and of the stack.
// Declarations and the contract of every entry point are in zaya.h.
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "zaya.h"

namespace zaya {

int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

namespace {

// ------------------------------------------------------------------ stage timing
// Optional: a CUDA event pair recorded around every kernel launch of a block
// on the caller's stream, accumulated per stage name.
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
  int kernels;
};
struct ProfAcc {
  const char* name;
  double ms;
  int64_t launches;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_pending;
std::vector<ProfAcc> g_prof_acc;
std::vector<cudaEvent_t> g_prof_pool;
std::atomic<int64_t> g_launches{0};

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct StageScope {
  const char* name;
  int kernels;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  StageScope(const char* n, int k, cudaStream_t s) : name(n), kernels(k), st(s) {
    if (g_prof_on) {
      std::lock_guard<std::mutex> lk(g_prof_mu);
      a = prof_event();
      cudaEventRecord(a, st);
    }
  }
  ~StageScope() {
    g_launches += kernels;
    if (a) {
      std::lock_guard<std::mutex> lk(g_prof_mu);
      cudaEvent_t b = prof_event();
      cudaEventRecord(b, st);
      g_prof_pending.push_back({name, a, b, kernels});
    }
  }
};

#define ZAYA_STAGE(name, nk, call)        \
  do {                                    \
    StageScope _sc((name), (nk), st);     \
    int _rc = (call);                     \
    if (_rc != ZAYA_OK) return _rc;       \
  } while (0)

constexpr size_t kAlign = 256;
inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Derived {
  int H, nq, nkv, d, C, n_qkv, qd, E, E1, I, R;
  float scale;
};

Derived derive(const zaya_config& c) {
  Derived d;
  d.H = c.hidden;
  d.nq = c.n_q;
  d.nkv = c.n_kv;
  d.d = c.head_dim;
  d.qd = c.n_q * c.head_dim;
  d.C = (c.n_q + c.n_kv) * c.head_dim;
  d.n_qkv = d.qd + 2 * c.n_kv * c.head_dim;
  d.E = c.n_experts;
  d.E1 = c.n_experts + 1;
  d.I = c.inter;
  d.R = c.router_hidden;
  d.scale = c.attn_scale > 0.f ? c.attn_scale : 1.0f / sqrtf((float)c.head_dim);
  return d;
}

int check_config(const zaya_config* c) {
  if (!c) return ZAYA_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->n_q <= 0 || c->n_kv <= 0 || c->head_dim <= 0 || c->n_experts <= 0 || c->inter <= 0 ||
      c->router_hidden <= 0 || c->window <= 0 || c->rot_dim < 0)
    return ZAYA_ERR_INVALID_ARG;
  if (c->n_q % c->n_kv) return ZAYA_ERR_INVALID_ARG;
  if (c->conv_groups < 0) return ZAYA_ERR_INVALID_ARG;
  if (!((c->conv_width == 3 && c->conv_groups == 0) || (c->conv_width == 2 && c->conv_groups == c->n_q + c->n_kv)))
    return ZAYA_ERR_UNSUPPORTED;
  if (c->hidden % 128 || c->hidden > 4096) return ZAYA_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return ZAYA_ERR_UNSUPPORTED;
  if (c->rot_dim > c->head_dim || c->rot_dim % 2 || (c->rot_dim / 2) % (c->head_dim / 32)) return ZAYA_ERR_UNSUPPORTED;
  const int rep = c->n_q / c->n_kv;
  if (rep != 1 && rep != 2 && rep != 4 && rep != 8) return ZAYA_ERR_UNSUPPORTED;
  if (c->n_q + 2 * c->n_kv > 32) return ZAYA_ERR_UNSUPPORTED;
  if (c->n_experts > 64) return ZAYA_ERR_UNSUPPORTED;
  if (c->inter % 128) return ZAYA_ERR_UNSUPPORTED;
  if (c->router_hidden % 32 || c->router_hidden > 256) return ZAYA_ERR_UNSUPPORTED;
  if (c->rms_eps < 0.f || c->qk_norm_eps <= 0.f) return ZAYA_ERR_INVALID_ARG;
  if (c->sliding_period < 0 || (c->sliding_period > 0 && (c->sliding_phase < 0 || c->sliding_phase >= c->sliding_period)))
    return ZAYA_ERR_INVALID_ARG;
  // a window ring needs a window on every block
  if (c->kv_ring != 0 && (c->kv_ring != 1 || c->sliding_period > 0)) return ZAYA_ERR_INVALID_ARG;
  if (c->kv_fp8 != 0 && c->kv_fp8 != 1) return ZAYA_ERR_INVALID_ARG;
  if (c->expert_fp8 != 0 && c->expert_fp8 != 1) return ZAYA_ERR_INVALID_ARG;
  if (c->expert_fp8 && (c->inter % 128 || c->hidden % 256)) return ZAYA_ERR_UNSUPPORTED;   // swapped pair tiles
  return ZAYA_OK;
}

// Keys (its own included) a query of block `block_idx` attends over: the
// config's window, or every earlier token on the blocks a hybrid stack does
// not slide (a window no sequence of the library reaches).
constexpr int kFullWindow = 1 << 30;
int block_window(const zaya_config& c, int block_idx) {
  if (c.sliding_period <= 0 || block_idx % c.sliding_period == c.sliding_phase) return c.window;
  return kFullWindow;
}
// Most key chunks a decode step's attention uses over the config's blocks.
int decode_chunks_any(const zaya_config& c) {
  return decode_attn_max_chunks(c.sliding_period > 0 ? kFullWindow : c.window);
}
// Largest prefill attention workspace over the windows the config's blocks use.
size_t attn_prefill_ws_any(const zaya_config& c, int B, int S, int nq, int nkv, int d) {
  size_t n = attn_prefill_ws_bytes(B, S, c.window, nq, nkv, d);
  if (c.sliding_period > 0) {
    const size_t f = attn_prefill_ws_bytes(B, S, kFullWindow, nq, nkv, d);
    if (f > n) n = f;
  }
  return n;
}

inline bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_weights(const zaya_block_weights* w, const zaya_config* c) {
  if (!w) return ZAYA_ERR_INVALID_ARG;
  if (c->conv_groups > 0 && (!w->conv2_w || !w->conv2_b)) return ZAYA_ERR_INVALID_ARG;
  if (c->conv_groups > 0 && (!a16(w->conv2_w) || !a16(w->conv2_b))) return ZAYA_ERR_MISALIGNED;
  if (c->expert_fp8 && (!w->w_gate_up_scale || !w->w_down_scale || !w->expert_act_scale)) return ZAYA_ERR_INVALID_ARG;
  if (c->expert_fp8 && (!a16(w->w_gate_up_scale) || !a16(w->w_down_scale) || !a16(w->expert_act_scale)))
    return ZAYA_ERR_MISALIGNED;
  const void* ptrs[] = {w->ln1_w, w->ln2_w, w->w_qkv, w->conv_w, w->conv_b, w->k_temp, w->w_o, w->merge_a,
                        w->merge_m, w->router_down_w, w->router_down_b, w->router_state_scale, w->router_norm_w,
                        w->fc1_w, w->fc1_b, w->fc2_w, w->fc2_b, w->out_w, w->balancing, w->w_gate_up, w->w_down};
  for (const void* p : ptrs)
    if (!p) return ZAYA_ERR_INVALID_ARG;
  const void* mats[] = {w->ln1_w, w->ln2_w, w->w_qkv, w->w_o, w->router_down_w, w->w_gate_up, w->w_down,
                        w->merge_a, w->merge_m, w->out_w, w->fc1_w, w->fc2_w, w->conv_w, w->conv_b,
                        w->router_down_b, w->router_state_scale};
  for (const void* p : mats)
    if (!a16(p)) return ZAYA_ERR_MISALIGNED;
  return ZAYA_OK;
}

struct Ws {
  size_t status, a_in, qkv, q, premix, m_in, logits, cls, w, pos, perm, group_off, mt_start, xperm, act, part, rpart,
      wsplit, slot, ccount, convy, loany, kvlin, total;
};

Ws plan(const zaya_config& c, int mode, int B, int S) {
  const Derived d = derive(c);
  const size_t M = (size_t)B * (mode == ZAYA_DECODE ? 1 : S);
  const size_t rows_a = M + (mode == ZAYA_DECODE ? (size_t)B : 0);
  Ws w;
  size_t o = 0;
  w.status = o; o += up(256);
  w.a_in = o; o += up(rows_a * d.H * 2);
  w.qkv = o; o += up(rows_a * d.n_qkv * 2);
  w.q = o; o += up(M * d.qd * 2);
  w.premix = o; o += up(M * d.qd * 2);
  w.m_in = o; o += up(M * d.H * 2);
  w.logits = o; o += up(M * d.E1 * 4);
  w.cls = o; o += up(M * 4);
  w.w = o; o += up(M * 4);
  w.pos = o; o += up(M * 4);
  w.perm = o; o += up(M * 4);
  w.group_off = o; o += up((size_t)(d.E + 2) * 4);
  w.mt_start = o; o += up((size_t)(d.E + 2) * 4);
  w.xperm = o; o += up(M * d.H * 2);
  w.act = o; o += up(M * d.I * 2);
  w.part = o; o += up(mode == ZAYA_DECODE ? decode_attn_ws_bytes(B, d.nq, d.d, decode_chunks_any(c))
                                           : attn_prefill_ws_any(c, B, S, d.nq, d.nkv, d.d));
  w.rpart = o; o += up((size_t)router_down_splits((int)M, d.R, d.H) * M * d.R * 4);
  w.wsplit = o; o += up(((size_t)4 * d.R * d.R + (size_t)2 * ((d.E + 1 + 7) / 8 * 8) * d.R) * 2);   // fc1, fc2, out_proj hi / lo
  w.slot = o; o += up(M * 4);
  w.ccount = o; o += up((size_t)(d.E + 2) * 4);
  w.convy = o; o += c.conv_groups > 0 ? up(M * d.C * 4) : 0;   // the two-stage conv's output (fp32)
  w.loany = o; o += up((size_t)router_split_blocks(d.R, d.E) * 4);
  // window-ring or fp8-cache prefill: the prompt's bf16 K and V ([B, n_kv, S, d]
  // each) for the attention, stored into the cache afterwards
  w.kvlin = o; o += ((c.kv_ring || c.kv_fp8) && mode == ZAYA_PREFILL) ? 2 * up(M * d.nkv * d.d * 2) : 0;
  w.total = o;
  return w;
}

template <class T>
inline T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

// Tile width for a persistent GEMM.  128-wide tiles measured fastest for the
// block's prefill contractions (q/k/v, o_proj + merge, expert down + merge:
// against 256 they trade a little operand reuse for a deeper TMA ring, twice
// the tiles to balance and half the exposed epilogue); when 128-wide tiles
// do not give every SM a tile (decode-sized M), the narrowest candidate does
// the most to spread the weight stream over the SMs.
constexpr int kPairMinRows = 1024;   // rows from which the GEMMs use CTA pairs (cta_group::2)
constexpr int kPairDenseBn = 128;    // tile width of the CTA-pair dense GEMMs (256 x 128 tiles)

int pick_bn_tiles(long m_tiles, int N, const int* cands, int n, int sms) {
  bool has128 = false;
  int narrow = 0;
  for (int i = 0; i < n; ++i) {
    if (N % cands[i]) continue;
    if (cands[i] == 128) has128 = true;
    if (!narrow || cands[i] < narrow) narrow = cands[i];
  }
  if (has128 && m_tiles * (N / 128) >= sms) return 128;
  return narrow;
}
int pick_bn(int M, int N, const int* cands, int n, int sms) {
  return pick_bn_tiles((M + 127) / 128, N, cands, n, sms);
}

// RoPE inverse frequencies theta^(-2i/rot) rounded to fp32 (Llama's rotary
// keeps them in fp32), computed once per call on the host.
void fill_inv_freq(float* out, int rot, float theta) {
  for (int i = 0; i < 64; ++i) out[i] = (2 * i < rot) ? (float)(1.0 / pow((double)theta, (double)(2 * i) / rot)) : 0.f;
}

#define ZAYA_TRY(x)            \
  do {                         \
    int _rc = (x);             \
    if (_rc != ZAYA_OK) return _rc; \
  } while (0)

// The block after the attention inputs are in place (both modes share it):
// o_proj + merge 1, norm, router, permutation, experts + merge 2.
int block_tail(const zaya_config& c, const Derived& d, const zaya_block_weights* w, int block_idx, int M,
               float* hidden, const float* rin, float* rout, const zaya_taps* taps, void* ws, const Ws& L,
               int* cache_len_inc, const int32_t* attn_mask, int sms, cudaStream_t st) {
  int* status = at<int>(ws, L.status);
  // o_proj with merge 1 fused: hidden <- layer_mid
  {
    GemmParams p{};
    p.M = M; p.N = d.H; p.K = d.qd; p.status = status;
    p.stream = hidden; p.merge = w->merge_a;
    p.tap_bf16 = taps ? taps->attention_output : nullptr;
    p.tap_f32 = taps ? taps->layer_mid : nullptr;
    const int c3[] = {256, 128, 64};
    const int bn = pick_bn(M, d.H, c3, 3, sms);   // single-CTA tiles measured faster here than pairs
    ZAYA_STAGE("o_proj_merge", 1, launch_gemm(EPI_MERGE_ATTN, bn, at<void>(ws, L.premix), M, w->w_o, d.H, p, sms, st));
  }
  void* m_in = at<void>(ws, L.m_in);
  ZAYA_STAGE("rmsnorm_mlp", 1, launch_rmsnorm(hidden, 1, 0, w->ln2_w, m_in, taps ? taps->mlp_norm_output : nullptr,
                                              M, d.H, c.rms_eps, nullptr, 0, st));
  int* cls = at<int>(ws, L.cls);
  float* wgt = at<float>(ws, L.w);
  float* rpart = at<float>(ws, L.rpart);
  const int ks = router_down_splits(M, d.R, d.H);
  if (ks == 0) {  // router down_proj + bias + carried state in one pass, straight into the state out
    GemmParams p{};
    p.M = M; p.N = d.R; p.K = d.H; p.status = status;
    p.out = rout; p.ldo = d.R; p.bias = w->router_down_b;
    p.prev = (block_idx > 0) ? rin : nullptr; p.prev_scale = w->router_state_scale;
    ZAYA_STAGE("router_down", 1, launch_gemm(EPI_ROUTER_DOWN, 64, m_in, M, w->router_down_w, d.R, p, sms, st));
  } else {  // router down_proj as fp32 partial sums over K slabs
    GemmParams p{};
    p.M = M; p.N = d.R; p.K = d.H; p.k_splits = ks; p.status = status;
    p.out = rpart; p.ldo = d.R;
    const int bn = (d.R % 256 == 0) ? 256 : (d.R % 128 == 0) ? 128 : (d.R % 64 == 0) ? 64 : 32;
    ZAYA_STAGE("router_down", 1, launch_gemm(EPI_STORE_F32, bn, m_in, M, w->router_down_w, d.R, p, sms, st));
  }
  {  // router state (slab sum + bias + carried state, unless fused above), router MLP, scoring, top-1
    RouterParams p{};
    p.part = rpart; p.n_splits = ks; p.bias = w->router_down_b;
    p.prev = (block_idx > 0) ? rin : nullptr; p.prev_scale = w->router_state_scale; p.r_out = rout;
    p.norm_w = w->router_norm_w;
    p.fc1_w = w->fc1_w; p.fc1_b = w->fc1_b; p.fc2_w = w->fc2_w; p.fc2_b = w->fc2_b;
    p.wsplit = at<__nv_bfloat16>(ws, L.wsplit);
    p.out_w = w->out_w; p.balancing = w->balancing; p.mask = attn_mask;
    p.logits = (taps && taps->router_logits) ? taps->router_logits : at<float>(ws, L.logits);
    p.cls = cls; p.idx = taps ? taps->expert_indices : nullptr; p.w = wgt;
    p.w_tap = taps ? taps->expert_weights : nullptr;
    p.M = M; p.R = d.R; p.E = d.E; p.eps = c.rms_eps;
    p.class_count = at<int>(ws, L.ccount); p.slot = at<int>(ws, L.slot); p.status = status;
    p.lo_any = at<int>(ws, L.loany); p.n_lo_words = router_split_blocks(d.R, d.E);
    ZAYA_STAGE("router_mlp", 2, launch_router(p, st));
  }
  int* group_off = at<int>(ws, L.group_off);
  int* mt_start = at<int>(ws, L.mt_start);
  int* pos = at<int>(ws, L.pos);
  int* perm = at<int>(ws, L.perm);
  // the expert GEMMs run swapped on CTA pairs (256 weight rows x each expert's
  // tokens, rounded to 16) whenever the widths allow: I a multiple of 128, H of 256
  const int pair = (d.I % 128 == 0 && d.H % 256 == 0) ? 1 : 0;
  void* xperm = at<void>(ws, L.xperm);
  {  // the token -> expert-row permutation, the copy of routed rows, merge 2 of skipped rows
    DispatchParams p{};
    p.cls = cls; p.class_count = at<int>(ws, L.ccount); p.slot = at<int>(ws, L.slot);
    p.pos = pos; p.perm = perm; p.group_off = group_off; p.mt_start = mt_start; p.tile_rows = pair ? 256 : 128;
    p.m_in = m_in; p.x_perm = xperm; p.stream = hidden; p.merge_m = w->merge_m;
    p.in_scale = c.expert_fp8 ? w->expert_act_scale : nullptr;
    p.tap_mlp_out = taps ? taps->mlp_output : nullptr;
    p.cache_len_inc = cache_len_inc;
    p.status = status;
    p.M = M; p.H = d.H; p.E = d.E;
    ZAYA_STAGE("dispatch", 1, launch_dispatch(p, st));
  }
  void* act = at<void>(ws, L.act);
  {  // experts: gate/up + SwiGLU
    GemmParams p{};
    p.M = M; p.N = d.I; p.K = d.H; p.grouped = 1; p.group_off = group_off; p.mt_start = mt_start;
    p.n_groups = d.E; p.b_rows_per_group = 2 * d.I; p.status = status; p.pair = pair;
    p.out = act; p.ldo = d.I;
    p.fp8 = c.expert_fp8; p.w_scale = w->w_gate_up_scale; p.act_scale = w->expert_act_scale;
    ZAYA_STAGE("experts_gate_up", 1, launch_gemm(EPI_SWIGLU, 256, xperm, M, w->w_gate_up, d.E * 2 * d.I, p, sms, st));
  }
  {  // experts: down + weight + merge 2, scattered back to token rows
    GemmParams p{};
    p.M = M; p.N = d.H; p.K = d.I; p.grouped = 1; p.group_off = group_off; p.mt_start = mt_start;
    p.n_groups = d.E; p.b_rows_per_group = d.H; p.status = status; p.pair = pair;
    p.stream = hidden; p.merge = w->merge_m; p.perm = perm; p.row_w = wgt;
    p.tap_bf16 = taps ? taps->mlp_output : nullptr;
    p.fp8 = c.expert_fp8; p.w_scale = w->w_down_scale; p.act_scale = w->expert_act_scale;
    const int c2[] = {256, 128};
    const int bn = pair ? (d.H % 256 == 0 ? 256 : 128) : pick_bn_tiles((M + 127) / 128 + d.E / 2, d.H, c2, 2, sms);
    ZAYA_STAGE("experts_down_merge", 1, launch_gemm(EPI_MERGE_MLP, bn, act, M, w->w_down, d.E * d.H, p, sms, st));
  }
  return ZAYA_OK;
}

int check_state(const zaya_block_state* s, int need_cap) {
  if (!s || !s->k_cache || !s->v_cache || !s->cache_len || !s->conv_state || !s->prev_hs) return ZAYA_ERR_INVALID_ARG;
  if (s->cache_cap < need_cap) return ZAYA_ERR_INVALID_ARG;
  if (!a16(s->k_cache) || !a16(s->v_cache) || !a16(s->conv_state) || !a16(s->prev_hs)) return ZAYA_ERR_MISALIGNED;
  return ZAYA_OK;
}

int block_prefill_impl(const zaya_config* cfg, const zaya_block_weights* w, int block_idx, int B, int S,
                       float* hidden, const int32_t* mask, const float* rin, float* rout, const zaya_block_state* state,
                       const zaya_taps* taps, void* ws, size_t ws_bytes, cudaStream_t st) {
  ZAYA_TRY(check_config(cfg));
  ZAYA_TRY(check_weights(w, cfg));
  if (B <= 0 || S <= 0 || !hidden || !rout || !ws) return ZAYA_ERR_INVALID_ARG;
  if (block_idx < 0 || (block_idx > 0 && !rin) || rin == rout) return ZAYA_ERR_INVALID_ARG;
  // a window ring holds any prompt's last cache_cap positions, and at least a window
  ZAYA_TRY(check_state(state, cfg->kv_ring ? block_window(*cfg, block_idx) : S));
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) || !a16(hidden) || !a16(rout)) return ZAYA_ERR_MISALIGNED;
  if (taps && taps->attention_queries && !a16(taps->attention_queries)) return ZAYA_ERR_MISALIGNED;
  const zaya_config& c = *cfg;
  const Derived d = derive(c);
  const Ws L = plan(c, ZAYA_PREFILL, B, S);
  if (ws_bytes < L.total) return ZAYA_ERR_WORKSPACE;
  const int M = B * S;
  const int sms = num_sms_current();
  const int window = block_window(c, block_idx);
  int* status = at<int>(ws, L.status);
  void* a_in = at<void>(ws, L.a_in);
  void* qkv = at<void>(ws, L.qkv);
  // K / V of the prompt for the attention: the caches themselves, or, for a
  // window ring or an fp8 cache, bf16 linear copies in the workspace, stored
  // into the cache after the attention
  const bool via_ws = c.kv_ring || c.kv_fp8;
  void* kc = state->k_cache;
  void* vc = state->v_cache;
  int kcap = state->cache_cap;
  if (via_ws) {
    kc = at<void>(ws, L.kvlin);
    vc = at<uint8_t>(ws, L.kvlin) + up((size_t)M * d.nkv * d.d * 2);
    kcap = S;
  }
  ZAYA_STAGE("rmsnorm_attn", 1, launch_rmsnorm(hidden, 1, 0, w->ln1_w, a_in,
                                               taps ? taps->attention_norm_output : nullptr, M, d.H, c.rms_eps,
                                               nullptr, 0, st));
  {
    GemmParams p{};
    p.M = M; p.N = d.n_qkv; p.K = d.H; p.status = status; p.out = qkv; p.ldo = d.n_qkv;
    const int c3[] = {256, 128, 64};
    p.pair = (M >= kPairMinRows && d.n_qkv % kPairDenseBn == 0) ? 1 : 0;
    const int bn = p.pair ? kPairDenseBn : pick_bn(M, d.n_qkv, c3, 3, sms);
    if (!bn) return ZAYA_ERR_UNSUPPORTED;
    ZAYA_STAGE("qkv_gemm", 1, launch_gemm(EPI_STORE_BF16, bn, a_in, M, w->w_qkv, d.n_qkv, p, sms, st));
  }
  if (c.conv_groups > 0) {
    ConvGroupedParams p{};
    p.qkv = qkv; p.ld = d.n_qkv; p.dw = w->conv_w; p.db = w->conv_b; p.gw = w->conv2_w; p.gb = w->conv2_b;
    p.mask = mask; p.y = at<float>(ws, L.convy); p.rows = M; p.S = S; p.C = d.C; p.decode = 0;
    ZAYA_STAGE("conv_grouped", 1, launch_conv_grouped(p, c.conv_groups, d.d, sms, st));
  }
  {
    CcaParams p{};
    p.conv_y = c.conv_groups > 0 ? at<float>(ws, L.convy) : nullptr;
    p.qkv = qkv; p.n_qkv = d.n_qkv; p.conv_w = w->conv_w; p.conv_b = w->conv_b; p.k_temp = w->k_temp;
    p.mask = mask; p.q_out = at<void>(ws, L.q); p.tap_q = taps ? taps->attention_queries : nullptr;
    p.k_cache = kc; p.v_cache = vc; p.cache_cap = kcap;
    p.cache_len = state->cache_len; p.conv_state = state->conv_state; p.prev_hs = state->prev_hs; p.a_in = a_in;
    p.B = B; p.S = S; p.H = d.H; p.n_q = d.nq; p.n_kv = d.nkv; p.d = d.d; p.rot = c.rot_dim;
    p.cca_res = c.cca_mean_residual; p.v_delayed = c.v_delayed; p.theta = c.rope_theta; p.eps = c.qk_norm_eps;
    p.decode = 0; p.status = status;
    size_t ctr_off = 0;   // the attention's split merge counters, cleared by this kernel
    p.n_zero_words = attn_prefill_ctr(B, S, window, d.nq, d.d, &ctr_off);
    p.zero_words = p.n_zero_words ? reinterpret_cast<int*>(at<uint8_t>(ws, L.part) + ctr_off) : nullptr;
    fill_inv_freq(p.inv_freq, c.rot_dim, c.rope_theta);
    ZAYA_STAGE("cca", 1, launch_cca(p, st));
  }
  {
    AttnParams p{};
    p.ctr_cleared = 1;
    p.q = at<void>(ws, L.q); p.k_cache = kc; p.v_cache = vc; p.mask = mask;
    p.out = at<void>(ws, L.premix);
    p.B = B; p.S = S; p.cap = kcap; p.n_q = d.nq; p.n_kv = d.nkv; p.d = d.d; p.window = window;
    p.scale = d.scale;
    p.part = at<void>(ws, L.part);
    p.part_bytes = attn_prefill_ws_bytes(B, S, window, d.nq, d.nkv, d.d);
    ZAYA_STAGE("attention", 1, launch_attn_prefill_tc(p, status, st));
  }
  if (via_ws)
    ZAYA_STAGE("cache_store", 1, launch_cache_store(kc, vc, state->k_cache, state->v_cache, B, d.nkv, S,
                                                    state->cache_cap, d.d, c.kv_ring, c.kv_fp8, status, st));
  return block_tail(c, d, w, block_idx, M, hidden, rin, rout, taps, ws, L, nullptr, mask, sms, st);
}

// Every host-side check of a decode call except the workspace's (shared with
// the entry point without a caller workspace, which runs them before it
// enqueues anything).
int check_decode_args(const zaya_config* cfg, const zaya_block_weights* w, int block_idx, int B, const float* hidden,
                      const float* rin, const float* rout, const zaya_block_state* state, const zaya_taps* taps) {
  ZAYA_TRY(check_config(cfg));
  ZAYA_TRY(check_weights(w, cfg));
  if (B <= 0 || !hidden || !rout) return ZAYA_ERR_INVALID_ARG;
  if (block_idx < 0 || (block_idx > 0 && !rin) || rin == rout) return ZAYA_ERR_INVALID_ARG;
  ZAYA_TRY(check_state(state, cfg->kv_ring ? block_window(*cfg, block_idx) : 1));
  if (!a16(hidden) || !a16(rout)) return ZAYA_ERR_MISALIGNED;
  if (taps && taps->attention_queries && !a16(taps->attention_queries)) return ZAYA_ERR_MISALIGNED;
  return ZAYA_OK;
}

int block_decode_impl(const zaya_config* cfg, const zaya_block_weights* w, int block_idx, int B, float* hidden,
                      const float* rin, float* rout, const zaya_block_state* state, const zaya_taps* taps, void* ws,
                      size_t ws_bytes, cudaStream_t st) {
  ZAYA_TRY(check_decode_args(cfg, w, block_idx, B, hidden, rin, rout, state, taps));
  if (!ws) return ZAYA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) return ZAYA_ERR_MISALIGNED;
  const zaya_config& c = *cfg;
  const Derived d = derive(c);
  const Ws L = plan(c, ZAYA_DECODE, B, 1);
  if (ws_bytes < L.total) return ZAYA_ERR_WORKSPACE;
  const int M = B;
  const int sms = num_sms_current();
  int* status = at<int>(ws, L.status);
  void* a_in = at<void>(ws, L.a_in);
  void* qkv = at<void>(ws, L.qkv);
  // rows [0,B): attention_norm_output; rows [B,2B): prev_hs (its projection gives the delayed values)
  ZAYA_STAGE("rmsnorm_attn", 1, launch_rmsnorm(hidden, 1, 0, w->ln1_w, a_in,
                                               taps ? taps->attention_norm_output : nullptr, M, d.H, c.rms_eps,
                                               state->prev_hs, B, st));
  {
    GemmParams p{};
    p.M = 2 * B; p.N = d.n_qkv; p.K = d.H; p.status = status; p.out = qkv; p.ldo = d.n_qkv;
    const int c3[] = {256, 128, 64};
    const int bn = pick_bn(2 * B, d.n_qkv, c3, 3, sms);
    if (!bn) return ZAYA_ERR_UNSUPPORTED;
    ZAYA_STAGE("qkv_gemm", 1, launch_gemm(EPI_STORE_BF16, bn, a_in, 2 * B, w->w_qkv, d.n_qkv, p, sms, st));
  }
  if (c.conv_groups > 0) {
    ConvGroupedParams p{};
    p.qkv = qkv; p.ld = d.n_qkv; p.dw = w->conv_w; p.db = w->conv_b; p.gw = w->conv2_w; p.gb = w->conv2_b;
    p.conv_state = state->conv_state; p.y = at<float>(ws, L.convy); p.rows = B; p.S = 1; p.C = d.C; p.decode = 1;
    ZAYA_STAGE("conv_grouped", 1, launch_conv_grouped(p, c.conv_groups, d.d, sms, st));
  }
  {
    CcaParams p{};
    p.conv_y = c.conv_groups > 0 ? at<float>(ws, L.convy) : nullptr;
    p.qkv = qkv; p.n_qkv = d.n_qkv; p.conv_w = w->conv_w; p.conv_b = w->conv_b; p.k_temp = w->k_temp;
    p.mask = nullptr; p.q_out = at<void>(ws, L.q); p.tap_q = taps ? taps->attention_queries : nullptr;
    p.k_cache = state->k_cache; p.v_cache = state->v_cache; p.cache_cap = state->cache_cap;
    p.cache_len = state->cache_len; p.conv_state = state->conv_state; p.prev_hs = state->prev_hs; p.a_in = a_in;
    p.B = B; p.S = 1; p.H = d.H; p.n_q = d.nq; p.n_kv = d.nkv; p.d = d.d; p.rot = c.rot_dim;
    p.cca_res = c.cca_mean_residual; p.v_delayed = c.v_delayed; p.theta = c.rope_theta; p.eps = c.qk_norm_eps;
    p.decode = 1; p.ring = c.kv_ring; p.fp8 = c.kv_fp8; p.status = status;
    fill_inv_freq(p.inv_freq, c.rot_dim, c.rope_theta);
    ZAYA_STAGE("cca", 1, launch_cca(p, st));
  }
  {
    DecodeAttnParams p{};
    p.q = at<void>(ws, L.q); p.k_cache = state->k_cache; p.v_cache = state->v_cache; p.cache_len = state->cache_len;
    p.out = at<void>(ws, L.premix); p.part = at<float>(ws, L.part);
    const int window = block_window(c, block_idx);
    p.B = B; p.cap = state->cache_cap; p.n_q = d.nq; p.n_kv = d.nkv; p.d = d.d; p.window = window;
    p.ring = c.kv_ring;
    p.fp8 = c.kv_fp8;
    const int span = window < state->cache_cap ? window : state->cache_cap;
    decode_attn_split(span, decode_chunks_any(c), &p.n_chunks, &p.chunk_keys);
    p.scale = d.scale;
    ZAYA_STAGE("attention_decode", 2, launch_attn_decode(p, st));
  }
  return block_tail(c, d, w, block_idx, M, hidden, rin, rout, taps, ws, L, state->cache_len, nullptr, sms, st);
}

}  // namespace
}  // namespace zaya

using namespace zaya;

extern "C" {

int zaya_abi_version(void) { return ZAYA_ABI_VERSION; }

const char* zaya_status_string(int code) {
  switch (code) {
    case ZAYA_OK: return "ok";
    case ZAYA_ERR_INVALID_ARG: return "invalid argument";
    case ZAYA_ERR_MISALIGNED: return "misaligned operand (16-byte alignment required)";
    case ZAYA_ERR_UNSUPPORTED: return "unsupported shape";
    case ZAYA_ERR_WORKSPACE: return "workspace too small";
    case ZAYA_ERR_CUDA: return "CUDA error";
    case ZAYA_ERR_TIMEOUT: return "device wait timed out";
    case ZAYA_ERR_DEVICE_RANGE: return "device index out of range";
    default: return "unknown status";
  }
}

size_t zaya_workspace_size(const zaya_config* cfg, int32_t mode, int32_t B, int32_t S) {
  if (check_config(cfg) != ZAYA_OK || B <= 0 || S <= 0 || (mode != ZAYA_PREFILL && mode != ZAYA_DECODE)) return 0;
  return plan(*cfg, mode, B, mode == ZAYA_DECODE ? 1 : S).total;
}

static size_t stack_extra(const zaya_config* cfg, int32_t mode, int32_t B, int32_t S, size_t* o_stream, size_t* o_r0,
                          size_t* o_r1, size_t* o_fn) {
  const size_t M = (size_t)B * (mode == ZAYA_DECODE ? 1 : S);
  size_t o = 0;
  *o_stream = o; o += up(M * cfg->hidden * 4);
  *o_r0 = o; o += up(M * cfg->router_hidden * 4);
  *o_r1 = o; o += up(M * cfg->router_hidden * 4);
  *o_fn = o; o += up(M * cfg->hidden * 2);
  return o;
}

size_t zaya_stack_workspace_size(const zaya_config* cfg, int32_t mode, int32_t B, int32_t S) {
  const size_t blk = zaya_workspace_size(cfg, mode, B, S);
  if (!blk) return 0;
  size_t a, b, c, d;
  return blk + stack_extra(cfg, mode, B, S, &a, &b, &c, &d);
}

int zaya_block_prefill(const zaya_config* cfg, const zaya_block_weights* w, int32_t block_idx, int32_t B, int32_t S,
                       float* hidden, const int32_t* attn_mask, const float* router_state_in, float* router_state_out,
                       const zaya_block_state* state, const zaya_taps* taps, void* workspace, size_t workspace_bytes,
                       void* stream) {
  return block_prefill_impl(cfg, w, block_idx, B, S, hidden, attn_mask, router_state_in, router_state_out, state, taps,
                            workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int zaya_block_decode(const zaya_config* cfg, const zaya_block_weights* w, int32_t block_idx, int32_t B, float* hidden,
                      const float* router_state_in, float* router_state_out, const zaya_block_state* state,
                      const zaya_taps* taps, void* workspace, size_t workspace_bytes, void* stream) {
  return block_decode_impl(cfg, w, block_idx, B, hidden, router_state_in, router_state_out, state, taps, workspace,
                           workspace_bytes, static_cast<cudaStream_t>(stream));
}

int zaya_stack_forward(const zaya_config* cfg, int32_t n_blocks, const zaya_block_weights* blocks, const void* embed,
                       const void* final_norm_w, int32_t mode, int32_t B, int32_t S, const int32_t* ids,
                       const int32_t* attn_mask, const zaya_block_state* states, void* logits, int32_t logits_last_only,
                       void* workspace, size_t workspace_bytes, void* stream) {
  ZAYA_TRY(check_config(cfg));
  if (n_blocks <= 0 || !blocks || !embed || !final_norm_w || !ids || !states || !logits || !workspace)
    return ZAYA_ERR_INVALID_ARG;
  if (mode != ZAYA_PREFILL && mode != ZAYA_DECODE) return ZAYA_ERR_INVALID_ARG;
  if (mode == ZAYA_DECODE) {
    S = 1;
    if (attn_mask) return ZAYA_ERR_INVALID_ARG;
  }
  if (B <= 0 || S <= 0 || cfg->vocab <= 0 || cfg->vocab % 64) return ZAYA_ERR_INVALID_ARG;
  if (!a16(embed) || !a16(final_norm_w) || !a16(logits)) return ZAYA_ERR_MISALIGNED;
  const size_t blk = zaya_workspace_size(cfg, mode, B, S);
  size_t o_stream, o_r0, o_r1, o_fn;
  const size_t extra = stack_extra(cfg, mode, B, S, &o_stream, &o_r0, &o_r1, &o_fn);
  if (workspace_bytes < blk + extra) return ZAYA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  void* bws = base;
  uint8_t* ex = base + blk;
  float* xs = reinterpret_cast<float*>(ex + o_stream);
  float* r[2] = {reinterpret_cast<float*>(ex + o_r0), reinterpret_cast<float*>(ex + o_r1)};
  void* fn = ex + o_fn;
  const int M = B * S;
  const Ws L = plan(*cfg, mode, B, S);
  int* status = reinterpret_cast<int*>(base + L.status);
  ZAYA_STAGE("embed", 1, launch_embed(ids, embed, xs, M, cfg->hidden, cfg->vocab, cfg->emb_mult, cfg->emb_shift, status, st));
  for (int i = 0; i < n_blocks; ++i) {
    const float* rin = i > 0 ? r[(i - 1) & 1] : nullptr;
    float* rout = r[i & 1];
    if (mode == ZAYA_PREFILL)
      ZAYA_TRY(zaya_block_prefill(cfg, &blocks[i], i, B, S, xs, attn_mask, rin, rout, &states[i], nullptr, bws, blk,
                                  stream));
    else
      ZAYA_TRY(zaya_block_decode(cfg, &blocks[i], i, B, xs, rin, rout, &states[i], nullptr, bws, blk, stream));
  }
  // final norm (all rows, or the last position of each sequence) + tied lm_head
  const bool last_only = mode == ZAYA_PREFILL && logits_last_only && S > 1;
  const int rows = last_only ? B : M;
  ZAYA_STAGE("final_norm", 1, launch_rmsnorm(xs, last_only ? S : 1, last_only ? S - 1 : 0, final_norm_w, fn, nullptr,
                                             rows, cfg->hidden, cfg->rms_eps, nullptr, 0, st));
  GemmParams p{};
  p.M = rows; p.N = cfg->vocab; p.K = cfg->hidden; p.status = status; p.out = logits; p.ldo = cfg->vocab;
  const int c3[] = {256, 128, 64};
  const int sms = num_sms_current();
  const int bn = pick_bn(rows, cfg->vocab, c3, 3, sms);
  if (!bn) return ZAYA_ERR_UNSUPPORTED;
  ZAYA_STAGE("lm_head", 1, launch_gemm(EPI_STORE_BF16, bn, fn, rows, embed, cfg->vocab, p, sms, st));
  return ZAYA_OK;
}

void zaya_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
}

void zaya_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof_pending) {
    cudaEventSynchronize(r.b);
    g_prof_pool.push_back(r.a);
    g_prof_pool.push_back(r.b);
  }
  g_prof_pending.clear();
  g_prof_acc.clear();
}

int zaya_profile_read(int32_t max_stages, const char** names, double* total_ms, int64_t* launches) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) ms = 0.f;
    ProfAcc* acc = nullptr;
    for (auto& x : g_prof_acc)
      if (strcmp(x.name, r.name) == 0) acc = &x;
    if (!acc) {
      g_prof_acc.push_back({r.name, 0.0, 0});
      acc = &g_prof_acc.back();
    }
    acc->ms += ms;
    acc->launches += 1;   // stage calls (a stage may launch more than one kernel)
    g_prof_pool.push_back(r.a);
    g_prof_pool.push_back(r.b);
  }
  g_prof_pending.clear();
  const int n = (int)g_prof_acc.size();
  for (int i = 0; i < n && i < max_stages; ++i) {
    if (names) names[i] = g_prof_acc[i].name;
    if (total_ms) total_ms[i] = g_prof_acc[i].ms;
    if (launches) launches[i] = g_prof_acc[i].launches;
  }
  return n;
}

int64_t zaya_launch_count(void) { return g_launches.load(); }

int zaya_device_status(void* workspace, void* stream) {
  if (!workspace) return ZAYA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ZAYA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ZAYA_ERR_CUDA;
  if (v != 0 && cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return ZAYA_ERR_CUDA;
  return v;
}

}  // extern "C"

// ------------------------------------------------------------------ decode without a caller workspace
// Scratch for zaya_block_decode_noalloc, in the library's own device memory:
// every GPU that loads this library holds these bytes until the process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (host code cannot use the symbol itself: on the host it names a
// host-side stand-in, not device memory).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZAYA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ZAYA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ZAYA_OK;
}
}  // namespace

extern "C" int zaya_block_decode_noalloc(const zaya_config* cfg, const zaya_block_weights* w, int32_t block_idx,
                                         int32_t B, float* hidden, const float* router_state_in,
                                         float* router_state_out, const zaya_block_state* state,
                                         const zaya_taps* taps, void* stream) {
  // every argument check first: an invalid call enqueues nothing
  ZAYA_TRY(check_decode_args(cfg, w, block_idx, B, hidden, router_state_in, router_state_out, state, taps));
  const size_t need = zaya_workspace_size(cfg, ZAYA_DECODE, B, 1);
  if (need == 0) return ZAYA_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return ZAYA_ERR_WORKSPACE;
  void* scratch = nullptr;
  ZAYA_TRY(noalloc_scratch(&scratch));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The scratch keeps the previous call's contents; only its 256-byte header
  // (the status word and the wait limit) must start at zero.
  if (cudaMemsetAsync(scratch, 0, 256, st) != cudaSuccess) return ZAYA_ERR_CUDA;
  return zaya_block_decode(cfg, w, block_idx, B, hidden, router_state_in, router_state_out, state, taps, scratch,
                           kNoAllocScratchBytes, stream);
}

extern "C" int zaya_noalloc_status(void* stream) {
  void* scratch = nullptr;
  ZAYA_TRY(noalloc_scratch(&scratch));
  return zaya_device_status(scratch, stream);
}
