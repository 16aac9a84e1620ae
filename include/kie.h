/*
 * kie.h -- C ABI of the batch-1 decode engine (libkie.so), NVIDIA B200 (sm_100a).
 *
 * What the library computes. The pages describe a persistent single-kernel
 * runtime: one GPU-resident program that runs the whole per-token decode step
 * (every matrix product, the attention, the normalisations and the token
 * choice) and hands each new token back to itself without returning control
 * to the CPU ("メモリの壁を打破する：標準的なGPUで
 * 3,000 tokens/sの推論を実現する", section "1. The Monokernel Runtime"; "Kog、より深い
 * GPU最適化でAI推論を高速化できると賭ける", section "KogがGPU推論の最適化をさらに
 * 深める理由"). At batch 1 the step is bound by streaming every active weight from
 * HBM once per token (same first page, section "ボトルネック：計算量ではなくメモリ
 * 帯域幅"), and launch, host-scheduling and synchronisation overheads are what the
 * persistent design removes (section "マイクロ秒が失われる場所").
 *
 * The model is a pre-norm decoder: RMSNorm, q/k/v projections, RoPE (half-split
 * pairs), causal attention over an fp16 KV cache, output projection + residual,
 * RMSNorm, SwiGLU MLP (or routed top-k SwiGLU experts plus a shared expert) +
 * residual, final RMSNorm, untied LM head and greedy argmax (lowest index on
 * exact ties). Weights are fp16; activations and accumulation are fp32.
 *
 * Conventions common to every call:
 *  - Every call is synchronous on the given stream: it returns after the work it
 *    queued has completed. `stream` is a cudaStream_t (NULL = legacy default).
 *  - One context serves one request on one GPU. Calls on one context are not
 *    thread-safe; distinct contexts are independent.
 *  - A device-side failure (a wait that ran past its deadline, a failed device
 *    check) poisons the context: every call except kie_reset, kie_destroy,
 *    kie_last_error, kie_position and kie_get_info then returns KIE_ERR_STATE.
 *  - On any error nothing of the failed call's effect on the context state
 *    (position, pending token) is kept, except that a poisoned context's KV
 *    cache contents are undefined until kie_reset.
 */
#ifndef KIE_H_
#define KIE_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct kie_ctx kie_ctx; /* opaque, owned by the library */

typedef enum {
  KIE_OK = 0,
  KIE_ERR_INVALID_ARG = -1,  /* bad pointer, size, shape, name or token id        */
  KIE_ERR_STATE = -2,        /* call out of order (decode before load, poisoned)  */
  KIE_ERR_CONTEXT_FULL = -3, /* position + tokens would exceed max_ctx            */
  KIE_ERR_CUDA = -4,         /* a CUDA runtime call failed (message in last_error) */
  KIE_ERR_TIMEOUT = -5,      /* a device-side wait gave up after its deadline     */
  KIE_ERR_DEVICE = -6,       /* a device-side check failed                        */
  KIE_ERR_OOM = -7           /* device or host allocation failed                  */
} kie_status;

/* Model shape. Dense models set n_experts = top_k = ffn_expert = ffn_shared = 0
 * and ffn > 0; MoE models set ffn = 0 and the expert fields; ffn_shared = 0 is
 * a MoE layer without a shared expert (its shared.* tensors are then not
 * passed to kie_load_weights). Each expert's rows are split over all CTAs, so
 * every routing decision loads every SM with the same bytes.
 * Constraints: d_model, n_heads*head_dim, ffn, ffn_expert, ffn_shared multiples
 * of 8; head_dim 64 or 128; each KV head serves 1 to 16 query heads (query
 * head h reads KV head floor(h * n_kv_heads / n_heads)), attended in equal
 * sub-units of at most 4 (a shape whose uneven groups would leave a sub-unit
 * empty is rejected); max_ctx >= 1.
 * Capacity of one launch (one CTA per SM, S SMs): the rows of every matrix are
 * split over the CTAs; a CTA keeps at most 64 residual rows (d_model <= 64 S,
 * checked by kie_create) and at most 1280 partial sums per phase (its rows of
 * the matrix times the matrix's column blocks of 512 or 768 inputs). The LM
 * head and the dense gate/up projection run in row chunks, so any vocabulary
 * and FFN width fit; the q/k/v, output and down projections and the MoE
 * phases must fit whole (at S = 148: down projection width up to about
 * 15,000). Each phase's whole input vector (the largest of d_model, n_heads *
 * head_dim and the FFN width; MoE: ffn_shared + top_k * ffn_expert) is held in
 * shared memory as fp32 beside the weight ring: about 40,000 values at most
 * (kie_create: "shape needs too much shared memory"). MoE: up to 256
 * experts, top_k up to 8, at most 192 CTAs. kie_load_weights and
 * kie_plan reject a shape past these bounds with KIE_ERR_INVALID_ARG ("a CTA
 * would hold N partial sums (max 1280)"). */
typedef struct {
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn, vocab;
  int32_t n_experts, top_k, ffn_expert, ffn_shared;
  int32_t max_ctx;
  float rms_eps;    /* RMSNorm: x / sqrt(mean(x^2) + rms_eps) * g            */
  float rope_theta; /* RoPE angle of pair i at position p: p * theta^(-2i/dh) */
} kie_config;

/* One weight tensor, fp16, row-major. Matrices are W[out, in] (y = W x):
 *   embed [V, d]; lm_head [V, d]; final_norm [d]
 *   layers.{l}.attn_norm [d]; .wq [hq*dh, d]; .wk, .wv [hk*dh, d]; .wo [d, hq*dh]
 *   layers.{l}.mlp_norm [d]
 *   dense: layers.{l}.w_gate, .w_up [ffn, d]; .w_down [d, ffn]
 *   MoE:   layers.{l}.router [E, d];
 *          layers.{l}.experts.{e}.w_gate, .w_up [ffe, d]; .w_down [d, ffe]
 *          layers.{l}.shared.w_gate, .w_up [ffs, d]; .w_down [d, ffs]
 * Vectors give shape {n, 1} or {1, n}. `on_device` = 1 means `data` is a device
 * pointer on the context's device (16-byte aligned), 0 a host pointer
 * (pageable or pinned). */
typedef struct {
  const char* name;
  const void* data;
  int64_t shape[2];
  int32_t on_device;
} kie_tensor;

/* Optional per-call controls of kie_decode (pass NULL for defaults). Every
 * pointer except trace_out may be host or device memory (detected per call),
 * caller-owned; device memory must belong to the context's device
 * (KIE_ERR_INVALID_ARG otherwise). */
typedef struct {
  const int32_t* forced_tokens; /* [n]: token fed back after step i; -1 = argmax.
                                   Used for teacher forcing; NULL = free run.   */
  float* logits_out;            /* [n][vocab] fp32 logits of every step; NULL = none */
  float* margins_out;           /* [n] top-1 minus second-largest logit; NULL = none */
  uint32_t timeout_ms;          /* deadline of every device-side wait; 0 = 1000 ms    */
  int32_t fault_cta;            /* test hook: this CTA skips its arrival at grid      */
  int32_t fault_barrier;        /*   barrier number fault_barrier; -1 = off           */
  uint64_t* trace_out;          /* device memory of the context's device,
                                   [grid][trace_cap][2] globaltimer stamps of each
                                   grid barrier's arrival and release; NULL = off */
  int32_t trace_cap;            /* barriers recorded per CTA                          */
  /* Token choice. temperature = 0 (the default): greedy argmax, lowest index
     on exact ties. temperature > 0: sampling inside the kernel -- z = logit /
     temperature; keep the top_k largest z (1 <= top_k <= 64; ties: lower
     index first); weights exp(z - max z); keep the shortest prefix, in that
     order, whose cumulative weight reaches top_p (0 < top_p <= 1) of the
     total; pick the first token whose cumulative weight exceeds u times the
     kept total. u = (w >> 8) * 2^-24, w the first output word of Philox4x32-10
     with counter (position of the step's forward, 0, 0, 0) and key (seed low
     32 bits, seed high 32 bits), so a split decode draws the same numbers.
     out_tokens gets the chosen token; margins_out still gets the top-1 minus
     top-2 logit. Errors: INVALID_ARG for a negative temperature, or, when
     sampling, top_k outside [1, 64] or top_p outside (0, 1]. */
  float temperature;
  int32_t top_k;
  float top_p;
  uint64_t seed;
} kie_decode_opts;

/* Static facts about a loaded context, for measurement. */
typedef struct {
  int32_t grid;               /* CTAs of the persistent launch (one per SM)            */
  int32_t threads;            /* threads per CTA                                      */
  int32_t n_stages;           /* shared-memory ring stages per CTA                    */
  int32_t stage_bytes;        /* bytes per ring stage                                 */
  int32_t smem_bytes;         /* dynamic shared memory per CTA                        */
  int32_t barriers_per_token; /* grid barriers per decoded token                      */
  int64_t stream_bytes;       /* weight bytes streamed per decoded token (dense: all
                                 matrices; MoE: router, shared and top_k experts),
                                 plus norm gains and one embedding row                */
  int64_t kv_bytes_per_pos;   /* K+V bytes read per cached position per token         */
  int64_t resident_bytes;     /* device bytes held by the packed weights              */
  int64_t launches;           /* kernels this context has launched so far             */
} kie_info;

/* Create a context on CUDA device `device`. Validates the shape, picks the
 * launch geometry and allocates the KV cache and scratch (no weights yet).
 * Errors: INVALID_ARG (shape), CUDA, OOM. On success *out owns the context. */
kie_status kie_create(const kie_config* cfg, int device, kie_ctx** out);

/* Copy and pack the model weights into library-owned device memory (the
 * phase-ordered, per-CTA weight tape). The caller keeps ownership of its
 * buffers and may free them when the call returns. All tensors named in the
 * kie_tensor comment must be given exactly once with the stated shapes. The
 * library also keeps row-major copies of the layer matrices for the prompt
 * path (about the model's size again in device memory).
 * May be called again to replace the weights; resets the position.
 * Errors: INVALID_ARG (missing/extra/misshapen tensor), CUDA, OOM. */
kie_status kie_load_weights(kie_ctx* ctx, const kie_tensor* tensors, int n_tensors,
                            void* stream);

/* Append `n` prompt tokens (host array, ids in [0, vocab)). Commits the pending
 * token (if any) and tokens[0..n-2] to the KV cache; tokens[n-1] becomes the
 * pending token. No logits are computed. The tokens run through the
 * tensor-core prompt path in chunks of up to 1024 (tcgen05 GEMMs with fused
 * epilogues, tensor-core attention over the cache; MoE: each routed expert
 * over its own tokens).
 * Errors: STATE (no weights / poisoned), INVALID_ARG, CONTEXT_FULL, CUDA,
 * TIMEOUT, DEVICE (a non-finite router logit). */
kie_status kie_prefill(kie_ctx* ctx, const int32_t* tokens, int n, void* stream);

/* Decode `n_tokens` tokens in ONE persistent launch. Step i forwards the pending
 * token at the current position, takes the greedy argmax, writes it to
 * out_tokens[i] (host or device, caller-owned, [n_tokens]) and makes it (or
 * forced_tokens[i] when >= 0) the pending token for step i+1.
 * Errors: STATE (no pending token, no weights, poisoned), INVALID_ARG,
 * CONTEXT_FULL (position + n_tokens > max_ctx; checked before launch), CUDA,
 * TIMEOUT (context poisoned), DEVICE (context poisoned). */
kie_status kie_decode(kie_ctx* ctx, int n_tokens, int32_t* out_tokens,
                      const kie_decode_opts* opts, void* stream);

/* Decode `n_tokens` tokens like kie_decode (free-running greedy, one persistent
 * launch), for callers that must not allocate device memory while they run:
 * for example a serving loop with a latency budget that cannot stall on the
 * driver's allocator (cudaMalloc may synchronise the device), or a component
 * that runs where all device memory belongs to another framework's pool.
 * There is no counterpart of this call in the paper; it is an integration aid.
 *
 * The call allocates nothing and frees nothing. The kernel's per-launch
 * scratch lives in a 512 KiB array in the library's device image, which every
 * GPU that loads the library holds until the process exits. Models whose
 * scratch (8 bytes per flagged value: two residual copies, q/k/v, attention
 * output, FFN hidden; plus attention partials) exceeds it are rejected with KIE_ERR_INVALID_ARG
 * and a message giving both sizes. `out_tokens` must be device memory of
 * the context's device ([n_tokens] int32, caller-owned); no logits, margins,
 * forced tokens or trace.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. Every call on every context of a device shares the one array:
 * calls whose work overlaps on the GPU race and give wrong results; issue
 * them one after another. Errors: as kie_decode, plus INVALID_ARG for an
 * `out_tokens` that is not memory of the context's device, or a model whose
 * scratch does not fit. */
kie_status kie_decode_static(kie_ctx* ctx, int n_tokens, int32_t* out_tokens, void* stream);

/* Truncate the sequence to its first `pos` committed positions (0 <= pos <=
 * current position) and make `pending` (in [0, vocab)) the token fed to the
 * next forward, e.g. to regenerate from a prefix. KV entries at positions >= pos
 * are simply overwritten by later calls. Host-side only, no GPU work.
 * Errors: INVALID_ARG, STATE (no weights, poisoned). */
kie_status kie_rewind(kie_ctx* ctx, int32_t pos, int32_t pending);

/* Rewind to an empty sequence: position 0, no pending token, error and poison
 * cleared. Keeps the weights and the KV allocation. */
kie_status kie_reset(kie_ctx* ctx);

/* Free every resource of the context. NULL is accepted. */
kie_status kie_destroy(kie_ctx* ctx);

/* Message of the last failed call on this context ("" if none). Valid until the
 * next call on the same context. NULL ctx gives the last kie_create failure. */
const char* kie_last_error(const kie_ctx* ctx);

/* Number of committed KV positions (tokens forwarded so far), or -1 for NULL. */
int32_t kie_position(const kie_ctx* ctx);

/* The pending token (fed to the next forward), or -1 if none / NULL ctx. */
int32_t kie_pending(const kie_ctx* ctx);

/* Fill *info for a context whose weights are loaded. Errors: INVALID_ARG, STATE. */
kie_status kie_get_info(const kie_ctx* ctx, kie_info* info);

/* Tile shape of one kind of matrix segment: K input columns cut into nk
 * column blocks of kc halves (K = nk * kc); a tile holds up to g rows of one
 * column block and is one bulk copy into a ring stage. */
typedef struct {
  int32_t K, g, nk, kc;
} kie_seg_shape;

/* One CTA's share of one matrix: rows [row0, row0 + nrows) of the matrix's
 * packed row order, stored at byte offset `off` of the weight tape (nrows * K
 * fp16 values as tiles of the kind's shape). Packed row order: q/k/v rows are
 * [wq; wk; wv] with each head's dims ordered 0, dh/2, 1, dh/2 + 1, ... (RoPE
 * pairs adjacent); gate/up rows alternate gate_0, up_0, gate_1, up_1, ...;
 * other matrices keep their own row order. */
typedef struct {
  int64_t off;
  int32_t row0, nrows;
} kie_seg_range;

typedef struct {
  int32_t slots;          /* ranges per layer: 4 dense; 4 + 2 * n_experts MoE      */
  int32_t ranges_per_cta; /* n_layers * slots + 1                                 */
  int64_t tape_bytes;     /* size of the packed weight tape                       */
  kie_seg_shape shapes[9]; /* by kind: 0 q/k/v, 1 o, 2 gate/up, 3 down, 4 shared
                              gate/up, 5 expert gate/up, 6 shared down, 7 expert
                              down, 8 LM head; kinds the model lacks are zero     */
} kie_plan_info;

/* The weight-tape plan the engine uses for `grid` CTAs with ring stages of
 * `stage_bytes` (kie_get_info reports both for a real context): tile shapes,
 * and per CTA c, layer l and slot s the range ranges[c * ranges_per_cta +
 * l * slots + s] (slot 0 q/k/v, 1 o, 2 gate/up or shared gate/up, 3 down or
 * shared down, 4 + e expert e's gate/up, 4 + E + e expert e's down), with the
 * LM head's range last. The tape holds each CTA's ranges contiguously in that
 * order; the o and down ranges of a CTA are the same residual rows in every
 * layer. Pure host arithmetic: needs no GPU and allocates no device memory.
 * `ranges` may be NULL (then only *info is filled); otherwise it is a
 * caller-owned array of `capacity` entries, at least grid * ranges_per_cta.
 * Errors: INVALID_ARG for a shape kie_create would reject, grid < 1,
 * stage_bytes < 4096 or not a multiple of 16, a plan that needs more
 * per-CTA partial sums than the kernel holds, or too small a capacity
 * (message from kie_last_error(NULL)). */
kie_status kie_plan(const kie_config* cfg, int32_t grid, int32_t stage_bytes, kie_plan_info* info,
                    kie_seg_range* ranges, int64_t capacity);

#ifdef __cplusplus
}
#endif

#endif /* KIE_H_ */
