/* zaya.h -- C ABI of the B200 (sm_100a) ZAYA1 decoder-block forward.
 *
 * What the block computes (nnterp encyclopedia, "zaya" family page, section
 * "The block, in order", and the family-module docstring):
 *
 *   h   = merge_a(self_attn(input_layernorm(x)), x)
 *   out = merge_m(mlp(post_attention_layernorm(h)), h)
 *   merge(o, r) = (o + hidden_states_bias) * hidden_states_scale
 *               + (r + residual_bias) * residual_scale
 *
 * self_attn is CCA-style attention (same page, "Queries and keys are
 * convolved, normed to sqrt(head_dim) and the keys scaled"): q/k/v
 * projections, a causal depthwise convolution of width 3 over the q||k
 * channels, the CCA mean residual, per-head L2 norm to sqrt(d) with a
 * per-kv-head key temperature, rotary on the first half of each head,
 * sliding-window grouped-query softmax attention and o_proj.  mlp is a top-1
 * mixture of SwiGLU experts chosen beside a skip class by a router whose
 * state carries from block to block (same page, "One expert per token,
 * chosen beside a skip class").  The stream is float32 whatever the load;
 * norms cast it to bf16 first (same page, "The stream is float32 whatever
 * the load").  The decode state per block is the KV cache plus
 * conv_state [B,1280,2] and prev_hs [B,2048] (ZAYA1-8B-JANGTQ2 README,
 * "Architecture Summary").
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the
 *    library allocates nothing and keeps no state between calls.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream); nothing synchronises the host.  The
 *    library's kernels are launched with programmatic stream serialisation:
 *    each may be scheduled while the previous kernel of the stream finishes,
 *    but touches global memory only after that kernel has completed, so the
 *    usual stream order holds for the caller's own work on the stream.
 *  - Row-major layouts; bf16 = IEEE bfloat16, fp32 = IEEE float.
 *  - Every weight matrix and vector of zaya_block_weights except k_temp,
 *    the router MLP biases and norm weight, and balancing, and every bf16
 *    activation, must start on a 16-byte boundary (ZAYA_ERR_MISALIGNED
 *    otherwise); every pointer must be non-NULL unless stated otherwise
 *    (ZAYA_ERR_INVALID_ARG).
 *  - Return value: ZAYA_OK (0) or a ZAYA_ERR_* code; argument errors are
 *    detected on the host before anything is launched.  Faults found on the
 *    device (a bounded wait that ran out, an index out of range) are written
 *    to a status word in the workspace and read with zaya_device_status().
 *  - The workspace starts with a 256-byte header: the status word (int32 at
 *    byte 0) and a wait limit (uint64 nanoseconds at byte 8; 0 means the
 *    default of 2 s, and a test may set a shorter one to make the bounded
 *    waits run out).  The header must be zero before the first call on a
 *    workspace (cudaMemsetAsync); the calls never clear it themselves, so a
 *    fault stays recorded across calls until zaya_device_status() reads and
 *    clears it.
 *  - Fail fast: once the status word holds a fault, the library's kernels
 *    that wait on asynchronous copies skip their work, and a wait gives up as
 *    soon as another has recorded a fault, so a failed call (or stack) ends
 *    within one wait limit.  The outputs of a call that recorded a fault are
 *    unspecified.
 */
#ifndef ZAYA_H_
#define ZAYA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZAYA_ABI_VERSION 3

enum zaya_status {
  ZAYA_OK = 0,
  ZAYA_ERR_INVALID_ARG = 1,  /* NULL pointer, bad shape or config value */
  ZAYA_ERR_MISALIGNED = 2,   /* a bf16 operand not 16-byte aligned */
  ZAYA_ERR_UNSUPPORTED = 3,  /* a shape these kernels are not built for */
  ZAYA_ERR_WORKSPACE = 4,    /* workspace smaller than zaya_workspace_size() */
  ZAYA_ERR_CUDA = 5,         /* a CUDA launch or runtime call failed */
  ZAYA_ERR_TIMEOUT = 6,      /* device: a bounded wait ran out */
  ZAYA_ERR_DEVICE_RANGE = 7  /* device: a computed index fell outside its buffer */
};

enum zaya_mode { ZAYA_PREFILL = 0, ZAYA_DECODE = 1 };

/* Shapes and every choice the pages leave open, passed by value.
 * Supported: hidden % 128 == 0 and <= 4096; head_dim in {64, 128};
 * rot_dim even and <= head_dim; n_q % n_kv == 0; conv_width == 3 with
 * conv_groups == 0, or conv_width == 2 with conv_groups == n_q + n_kv;
 * n_experts <= 64; inter % 128 == 0; router_hidden % 32 == 0 and <= 256. */
typedef struct zaya_config {
  int32_t hidden;            /* H (2048 on ZAYA1-8B) */
  int32_t n_q;               /* query heads (8) */
  int32_t n_kv;              /* key/value heads (2); query head h uses kv head h / (n_q/n_kv) */
  int32_t head_dim;          /* d (128) */
  int32_t rot_dim;           /* rotated dims per head, pairs (i, i + rot_dim/2) (64) */
  int32_t conv_width;        /* 3: one depthwise conv, taps over tokens (t-2, t-1, t);
                                2: the printout's two convs of width 2 (conv_groups > 0) */
  int32_t n_experts;         /* E (16); the router scores E + 1 classes, the last is skip */
  int32_t inter;             /* expert width I (2048) */
  int32_t router_hidden;     /* R (256) */
  int32_t window;            /* key j visible to query i iff 0 <= i - j < window */
  int32_t vocab;             /* stack only: embedding rows */
  int32_t cca_mean_residual; /* 1: add the CCA mean residual after the conv */
  int32_t v_delayed;         /* 1: second half of each value head from token t-1 */
  int32_t sliding_period;    /* 0: every block attends over `window` keys.  P > 0: only blocks with
                                block_idx % P == sliding_phase do; the others attend to every
                                earlier token (ZAYA1-74B-preview: a 4097-token window on every
                                other block; zaya page, "Queries and keys are convolved ...") */
  int32_t sliding_phase;     /* 0 <= sliding_phase < sliding_period */
  int32_t conv_groups;       /* 0: conv_w is the width-3 depthwise conv.  G > 0: conv_qk_depthwise
                                (k=2, conv_w [C,2], conv_b) then conv_qk_grouped (k=2, G groups,
                                conv2_w, conv2_b) as the zaya page's printout lists them; the
                                kernels take one group per q / k head (G = n_q + n_kv, 10 on ZAYA1-8B) */
  int32_t kv_ring;           /* 0: position p of a sequence in cache slot p (cache_cap bounds the
                                positions).  1: slot p % cache_cap, a window ring: decode needs
                                cache_cap >= window and keeps only the last cache_cap positions,
                                so a sequence decodes past cache_cap with a window-sized cache
                                (the pages' decode reads the window only: zaya page, "Queries and
                                keys are convolved ..."; every block must slide: sliding_period 0) */
  int32_t expert_fp8;        /* 1: the experts as an FP8 W8A8 checkpoint (the pages' deployments
                                quantise the experts: NVFP4 README, "Quantization
                                details"): E4M3 weight codes with per-row fp32 scales, inputs
                                quantised to E4M3 with static per-expert scales, products on the
                                tensor cores in E4M3 (tcgen05 kind::f8f6f4), fp32 accumulation;
                                needs inter % 128 == 0 and hidden % 256 == 0 */
  int32_t kv_fp8;            /* 0: the caches hold bf16 keys / values.  1: OCP FP8 E4M3 bytes (the
                                bf16 value rounded to nearest, ties to even, saturating at 448), as
                                a serving engine's fp8 KV cache (NVFP4 README, "Throughput and
                                memory": --kv-cache-dtype fp8); a prompt attends over its bf16
                                keys / values, a decode step over the cache */
  float rope_theta;          /* inv_freq[i] = rope_theta^(-2i/rot_dim) */
  float rms_eps;             /* RMSNorm epsilon (1e-5) */
  float qk_norm_eps;         /* q,k -> x * sqrt(d) / max(|x|, qk_norm_eps) */
  float attn_scale;          /* softmax scale; <= 0 means 1/sqrt(head_dim) */
  float emb_mult;            /* stack only: stream0 = fp32((E[id] + emb_shift) * emb_mult) */
  float emb_shift;
} zaya_config;

/* One block's parameters (device pointers, caller-owned).
 * Linear weights are [out, in] row-major like nn.Linear.  C = (n_q + n_kv) * d. */
typedef struct zaya_block_weights {
  const void* ln1_w;              /* bf16 [H]   input_layernorm weight */
  const void* ln2_w;              /* bf16 [H]   post_attention_layernorm weight */
  const void* w_qkv;              /* bf16 [n_q*d + n_kv*d + n_kv*d, H]: rows q_proj, k_proj,
                                     v_proj_current (n_kv*d/2 rows), v_proj_delayed (n_kv*d/2) */
  const float* conv_w;            /* fp32 [C, 3] taps for (t-2, t-1, t) over the q||k channels;
                                     with conv_groups > 0: [C, 2] depthwise taps for (t-1, t) */
  const float* conv_b;            /* fp32 [C] */
  const float* k_temp;            /* fp32 [n_kv] key temperature */
  const void* w_o;                /* bf16 [H, n_q*d] o_proj */
  const float* merge_a;           /* fp32 [4, H] rows: hidden_states_bias, hidden_states_scale,
                                     residual_bias, residual_scale (post_attention_residual_scale) */
  const float* merge_m;           /* fp32 [4, H] same, post_mlp_residual_scale */
  const void* router_down_w;      /* bf16 [R, H] router down_proj */
  const float* router_down_b;     /* fp32 [R] */
  const float* router_state_scale;/* fp32 [R] multiplies the previous block's router state */
  const float* router_norm_w;     /* fp32 [R] router_mlp.norm */
  const float* fc1_w;             /* fp32 [R, R] */
  const float* fc1_b;             /* fp32 [R] */
  const float* fc2_w;             /* fp32 [R, R] */
  const float* fc2_b;             /* fp32 [R] */
  const float* out_w;             /* fp32 [E+1, R] router_mlp.out_proj (no bias) */
  const float* balancing;         /* fp32 [E+1] balancing_biases (selection only) */
  const void* w_gate_up;          /* bf16 [E, 2I, H]: rows [0,I) gate, [I,2I) up
                                     (expert_fp8: E4M3 codes, uint8) */
  const void* w_down;             /* bf16 [E, H, I] (expert_fp8: E4M3 codes) */
  const float* conv2_w;           /* conv_groups > 0 only (else may be NULL): fp32 [C, C/G, 2]
                                     conv_qk_grouped taps for (t-1, t) of the depthwise output,
                                     Conv1d's [out, in/groups, k] layout */
  const float* conv2_b;           /* conv_groups > 0 only: fp32 [C] */
  const float* w_gate_up_scale;   /* expert_fp8 only (else may be NULL): fp32 [E, 2I], one scale per
                                     row of w_gate_up (weight = code value x scale); 16-byte aligned */
  const float* w_down_scale;      /* expert_fp8 only: fp32 [E, H], one per row of w_down */
  const float* expert_act_scale;  /* expert_fp8 only: fp32 [E, 2] static input scales, powers of two:
                                     [e][0] for mlp_norm_output into gate/up (x_q = E4M3(x / s)),
                                     [e][1] for the SwiGLU output into down */
} zaya_block_weights;

/* One block's decode state (in/out, caller-owned). */
typedef struct zaya_block_state {
  void* k_cache;        /* bf16 (kv_fp8: E4M3 bytes) [B, n_kv, cache_cap, d]: keys after norm,
                           temp and RoPE (this and the three state buffers below: 16-byte aligned) */
  void* v_cache;        /* bf16 (kv_fp8: E4M3 bytes) [B, n_kv, cache_cap, d] */
  int32_t cache_cap;    /* positions per sequence the caches hold */
  int32_t* cache_len;   /* device int32 [B]: prefill writes S; decode appends at cache_len[b]
                           and increments it */
  void* conv_state;     /* bf16 [B, C, 2]: pre-conv q||k of tokens t-2 ([...,0]) and t-1 ([...,1]) */
  void* prev_hs;        /* bf16 [B, H]: attention_norm_output of token t-1 */
} zaya_block_state;

/* Optional per-block outputs named as nnterp names them (any may be NULL).
 * M = B*S rows in prefill, B rows in decode. */
typedef struct zaya_taps {
  float* router_logits;      /* fp32 [M, E+1] */
  int32_t* expert_indices;   /* int32 [M]: chosen expert, 0 for skip */
  float* expert_weights;     /* fp32 [M]: softmax entry of the chosen class, 0 for skip */
  void* attention_norm_output;/* bf16 [M, H] */
  void* attention_output;    /* bf16 [M, H]: (o_proj(attn) + hb) * hs */
  float* layer_mid;          /* fp32 [M, H] */
  void* mlp_norm_output;     /* bf16 [M, H] */
  void* mlp_output;          /* bf16 [M, H]: (routed + hb) * hs */
  void* attention_queries;   /* bf16 [B, n_q, S, d] (prefill) / [B, n_q, d] (decode); 16-byte aligned */
} zaya_taps;

/* Bytes of device workspace a call needs: mode ZAYA_PREFILL with (B, S), or
 * ZAYA_DECODE with (B, 1).  zaya_stack_forward needs
 * zaya_stack_workspace_size().  Returns 0 for an invalid config. */
size_t zaya_workspace_size(const zaya_config* cfg, int32_t mode, int32_t B, int32_t S);
size_t zaya_stack_workspace_size(const zaya_config* cfg, int32_t mode, int32_t B, int32_t S);

/* One block over B fresh sequences of S tokens (zaya page, "The block, in
 * order").
 *  hidden           fp32 [B, S, H] in: layer_input; out: layer_output (in place).
 *  attn_mask        int32 [B, S] (1 = token, 0 = padding) or NULL (no padding).
 *                   Padding tokens take no part: their queries output 0,
 *                   keys at pads are masked, pads are routed to skip, and
 *                   their pre-conv q/k and delayed-value inputs are zero.
 *                   Positions are 0..S-1 for every sequence.
 *  block_idx        0 for the first block: the carried router state is not
 *                   added there (zaya page, "One expert per token ...").
 *  router_state_in  fp32 [B, S, R]; ignored when block_idx == 0, may then be NULL.
 *  router_state_out fp32 [B, S, R]: down_proj(mlp_norm_output) + bias
 *                   (+ router_state_in * router_state_scale); the next
 *                   block's router_state_in.  Must not alias router_state_in.
 *  state            K/V of every position written to the caches at 0..S-1
 *                   (cache_cap >= S); with kv_ring, the last min(S, cache_cap)
 *                   positions p at slots p % cache_cap (any S); with kv_ring
 *                   or kv_fp8 the attention reads the prompt's bf16 keys from
 *                   the workspace and a store kernel fills the cache; cache_len[b]
 *                   = S; conv_state and prev_hs set from the last two tokens.
 *                   Continuing a padded prefill in decode is not supported.
 *  taps             NULL or optional outputs.
 *  workspace        >= zaya_workspace_size(cfg, ZAYA_PREFILL, B, S) bytes,
 *                   256-byte aligned.  Its first word is the device status. */
int zaya_block_prefill(const zaya_config* cfg, const zaya_block_weights* w, int32_t block_idx,
                       int32_t B, int32_t S, float* hidden, const int32_t* attn_mask,
                       const float* router_state_in, float* router_state_out,
                       const zaya_block_state* state, const zaya_taps* taps,
                       void* workspace, size_t workspace_bytes, void* stream);

/* One new token for each of B sequences through a block with a cache.
 *  hidden fp32 [B, H] in/out.  router_state_in / _out fp32 [B, R].
 *  The token of sequence b sits at position cache_len[b]; it attends over
 *  positions max(0, t - window + 1) .. t; requires 0 <= cache_len[b] and,
 *  without kv_ring, cache_len[b] < cache_cap for every b (with kv_ring the
 *  token's K/V go to slot cache_len[b] % cache_cap, and cache_cap >= window
 *  is checked on the host), checked on the device: if any sequence fails it, the status
 *  word records ZAYA_ERR_DEVICE_RANGE and no sequence's caches, conv_state,
 *  prev_hs or cache_len are written (hidden and the router state out are
 *  then unspecified).
 *  conv_state, prev_hs, the caches and cache_len are updated. */
int zaya_block_decode(const zaya_config* cfg, const zaya_block_weights* w, int32_t block_idx,
                      int32_t B, float* hidden, const float* router_state_in, float* router_state_out,
                      const zaya_block_state* state, const zaya_taps* taps,
                      void* workspace, size_t workspace_bytes, void* stream);

/* zaya_block_decode without a caller-supplied workspace.  The paper has no
 * counterpart: this is a calling convention of the library.
 *
 * For callers that cannot allocate device memory where they run a decode
 * step -- for example a serving runtime that has handed all device memory to
 * its own pools and forbids further allocations, or a plain C host program
 * with no device allocator of its own -- and so cannot provide the workspace
 * zaya_block_decode takes.  Arguments and results are those of
 * zaya_block_decode; inputs and outputs are still the caller's buffers.
 *
 * Scratch: a fixed 8 MiB array in the library's own device memory (held on
 * every GPU that loads the library until the process exits), enough for a
 * full-width decode step (hidden 2048, 16 experts x 2048) of up to 64
 * sequences.  A call whose zaya_workspace_size(cfg, ZAYA_DECODE, B, 1)
 * exceeds 8 MiB returns ZAYA_ERR_WORKSPACE without launching anything.  No
 * cudaMalloc, cudaFree or other allocating call is made.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every argument is checked before anything is enqueued; an invalid
 *    call returns its ZAYA_ERR_* code with no GPU work issued.
 *  - All calls share the one array and it keeps the previous call's
 *    contents; each call first clears the array's 256-byte header (status
 *    word and wait limit) on `stream`.  Calls that overlap on the GPU (other
 *    streams, other threads) race on the array and corrupt each other:
 *    serialise them.
 *  - Device-side faults of the last call are recorded in the array's status
 *    word; zaya_noalloc_status() returns and clears it. */
int zaya_block_decode_noalloc(const zaya_config* cfg, const zaya_block_weights* w, int32_t block_idx, int32_t B,
                              float* hidden, const float* router_state_in, float* router_state_out,
                              const zaya_block_state* state, const zaya_taps* taps, void* stream);

/* Device status of zaya_block_decode_noalloc on the current device:
 * synchronises `stream`, returns the status word of the library's fixed
 * scratch (ZAYA_OK if none) and clears it.  Like the entry point it serves,
 * it has no counterpart on the pages. */
int zaya_noalloc_status(void* stream);

/* The whole stack: embedding -> n_blocks blocks (router state chained on the
 * device) -> final norm -> tied lm_head (zaya page, "Printout" and "The
 * readout and the tokenizer": logits = lm_head(norm(stream)), no cap).
 *  blocks      host array [n_blocks] of weight structs (device pointers inside).
 *  embed       bf16 [vocab, H]: embedding and lm_head weight.
 *  final_norm_w bf16 [H].
 *  mode        ZAYA_PREFILL (ids [B, S], fresh caches) or ZAYA_DECODE (ids [B], S = 1).
 *  attn_mask   as for zaya_block_prefill (prefill only; NULL for decode).
 *  states      host array [n_blocks] of state structs.
 *  logits      bf16 [B, S, vocab], or [B, vocab] when logits_last_only
 *              (the last position of each sequence) or in decode. */
int zaya_stack_forward(const zaya_config* cfg, int32_t n_blocks, const zaya_block_weights* blocks,
                       const void* embed, const void* final_norm_w, int32_t mode, int32_t B, int32_t S,
                       const int32_t* ids, const int32_t* attn_mask, const zaya_block_state* states,
                       void* logits, int32_t logits_last_only,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, returns the device status word recorded in
 * `workspace` (ZAYA_OK if none) and clears it. */
int zaya_device_status(void* workspace, void* stream);

/* Human-readable name of a status code (static storage). */
const char* zaya_status_string(int code);

/* Stage timing for measurement (no counterpart on the pages).  When enabled,
 * a CUDA event is recorded on the caller's stream before and after every
 * stage (one or two kernel launches) of the entry points above;
 * zaya_profile_read synchronises those events and returns, per stage name
 * (static strings such as "attention", "experts_gate_up"), the accumulated
 * milliseconds and the number of times the stage ran since the last reset.
 * Returns the number of stages, of which at most max_stages are written.
 * Off by default. */
void zaya_profile_enable(int on);
void zaya_profile_reset(void);
int zaya_profile_read(int32_t max_stages, const char** names, double* total_ms, int64_t* launches);

/* Number of CUDA kernels this library has launched since it was loaded. */
int64_t zaya_launch_count(void);

/* ZAYA_ABI_VERSION of the loaded library. */
int zaya_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ZAYA_H_ */
