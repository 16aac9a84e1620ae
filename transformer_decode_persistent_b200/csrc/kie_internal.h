// Internal layout shared by the host side (packer, launcher) and the
// persistent decode kernel. Not part of the public ABI (see include/kie.h).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace kie {

// ---- launch geometry ------------------------------------------------------
// 7 consumer warps + 1 producer warp = 256 threads: registers are allocated to
// a CTA in 4-warp steps, so 8 warps keep the 255-register ceiling that the
// attention sub-block loop needs (9 warps would be capped at 168 and spill).
constexpr int kConsumerWarps = 7;                      // GEMV / attention warps
constexpr int kConsumerThreads = kConsumerWarps * 32;  // named barrier 1 spans these
constexpr int kThreads = kConsumerThreads + 32;        // + one producer (TMA) warp
constexpr int kRingStages = 2 * kConsumerWarps;        // ring stages per CTA (2 per consumer warp)
constexpr int kMaxStageBytes = 16384;                  // upper bound of one stage (one weight tile)
constexpr int kMaxRowsPerTile = 8;                     // rows of one tile in general (register-blocked)
constexpr int kMaxRowsWide = 13;                       // rows of a tile 512 halves wide
constexpr int kPartFloats = 1280;                      // per-CTA partial-sum slots per phase
constexpr int kMaxHeadsPerGroup = 4;                   // query heads of one attention unit
constexpr int kMaxQueryHeadsPerKv = 16;                // query heads per KV head (GQA), in sub-units
constexpr int kMaxTopK = 8;                            // routed experts per token
constexpr int kAttnSub = 32;                           // positions per attention sub-block
constexpr int kMaxExperts = 256;
constexpr int kRouteMaxGrid = 192;                     // MoE: CTAs whose router partials one warp sums (3 pairs a lane)
constexpr int kMaxOwnRows = 64;                        // residual rows a CTA keeps in shared memory
constexpr int kSampleK = 64;                           // largest top-k of in-kernel sampling
constexpr int kSampleMaxGrid = 160;                    // CTAs whose candidates one CTA can merge

// ---- weight tape ------------------------------------------------------------
// The tape is one device buffer. CTA c owns a contiguous region holding, in
// execution order, its slice of every weight matrix of one decode step. A
// "segment" is one CTA's slice of one matrix: rows [row0, row0 + nrows) of the
// matrix's (virtual) row space, stored as groups of `g` rows (the last group
// may be shorter); each group is cut into `nk` column chunks of `kc` columns,
// and each (group, chunk) tile is stored row-major [g'][kc] and is one TMA
// bulk copy of g' * kc * 2 bytes.
enum SegKind : int {
  SK_QKV = 0,   // rows: [wq; wk; wv], K = d
  SK_O = 1,     // rows: wo, K = hq*dh
  SK_GU = 2,    // rows: gate_0, up_0, gate_1, up_1, ... (dense FFN), K = d
  SK_DOWN = 3,  // rows: w_down, K = ffn
  SK_SGU = 4,   // shared expert gate/up interleaved, K = d
  SK_EGU = 5,   // routed expert gate/up interleaved, K = d
  SK_SDOWN = 6, // shared expert down, K = ffs
  SK_EDOWN = 7, // routed expert down, K = ffe
  SK_LM = 8,    // lm_head, K = d
  SK_COUNT = 9
};

struct SegShape {
  int K;   // columns of the matrix (input length)
  int g;   // rows per tile (full groups)
  int nk;  // column chunks per group
  int kc;  // columns per chunk (K / nk, multiple of 8)
};

struct SegDesc {
  unsigned long long off;  // byte offset of this segment in the tape
  int row0;                // first (virtual) row owned by this CTA
  int nrows;               // rows owned (GU kinds: always even)
};

// Descriptor slots per layer: 0 QKV, 1 O, 2 GU|SGU, 3 DOWN|SDOWN,
// 4..4+E-1 EGU[e], 4+E..4+2E-1 EDOWN[e]. The LM head is slot 0 of layer L.
__host__ __device__ inline int slots_per_layer(int n_experts) { return 4 + 2 * n_experts; }

// ---- device control block ---------------------------------------------------
struct Ctrl {
  unsigned int arrive;   // grid barrier arrivals (monotonic within one launch)
  unsigned int abort;    // set to 1 by any CTA that gives up; all CTAs poll it
  int err;               // first error code (kie_status value), 0 = none
  int err_cta;           // CTA that recorded the error
  int err_step;          // decode step
  int err_where;         // 1 grid barrier, 2 ring full-wait, 3 ring empty-wait,
                         // 4 route wait, 5 device check, 6 flagged-word wait,
                         // 7 ring tile larger than a stage
  int final_token;       // pending token after the last step
  int pad;
};

struct Cand {  // per-CTA greedy candidate: best value, its index, second value
  float v1;
  int i1;
  float v2;
  int pad;
};

struct Params {
  // model shape
  int L, d, hq, hk, dh, ff, V, E, top_k, ffe, ffs, max_ctx;
  float eps;
  int qkv_rows;    // (hq + 2 hk) dh
  int slots;       // descriptor slots per layer
  // packed weights
  const unsigned char* tape;
  const SegDesc* desc;       // [grid][L * slots + 1]
  SegShape shp[SK_COUNT];
  const __half* embed;       // [V][d]
  const __half* attn_norm;   // [L][d]
  const __half* mlp_norm;    // [L][d]
  const __half* final_norm;  // [d]
  const __half* router;      // [L][E][d] (MoE) or null
  // state
  __half* kcache;            // [L][hk][max_ctx][dh]
  __half* vcache;
  const float2* rope;        // [max_ctx][dh/2] (cos, sin)
  // Flagged scratch, zeroed before every launch. Each 64-bit word holds a
  // float (low half) and the epoch of the phase that wrote it (high half);
  // words are written and read as single 64-bit accesses, so a reader that
  // sees the epoch it waits for also sees the value. Epoch of (step, layer l)
  // = 1 + step * (L + 1) + l; the LM head of a step uses layer index L.
  unsigned long long* fx;     // [2][d] residual stream after the output (0) / down (1) projection
  unsigned long long* fq;     // [hq*dh | hk*dh | hk*dh] rotated scaled q | this token's k | v (fp16-rounded)
  unsigned long long* fo;     // [hq*dh] attention output
  unsigned long long* fh;     // [hbuf] FFN hidden (dense: ff; MoE: ffs + top_k*ffe)
  unsigned long long* fcand;  // [grid][3] LM-head candidates: best value, its index, second value
  unsigned long long* apart;  // attention chunk records [hq][max_chunks][dh + 4]: (max, sum), pad, acc[dh]
  unsigned long long* froute; // MoE: router partials [E + 1][grid]: row e < E = this CTA's residual rows'
                              // share of router logit e (before the RMSNorm factor); row E = their sum of squares
  Ctrl* ctrl;
  int max_chunks;
  // run
  int pos0, n_steps, first_token, lm_from_step;
  const int* forced;         // device [n_steps] or null
  int* out_tokens;           // device [n_steps]
  float* logits_out;         // device [n_steps][V] or null
  float* margins_out;        // device [n_steps] or null
  unsigned long long timeout_ns;
  int fault_cta, fault_barrier;
  unsigned long long* trace; // device [grid][trace_cap][2] or null
  int trace_cap;
  // sampling (temperature > 0; greedy otherwise): top-k in [1, kSampleK],
  // top-p in (0, 1], Philox key `seed`. fsamp holds, flagged like the scratch
  // above, each CTA's local top-k as (value, index) word pairs [grid][2 *
  // kSampleK] and then the sampled token's word; cleared before a sampling launch.
  float samp_temp, samp_p;
  int samp_k;
  unsigned long long samp_seed;
  unsigned long long* fsamp;
  float* lm_logits;           // sampling: this step's LM-head logits of each CTA's rows [grid][lm_rows]
  int lm_rows;
  int n_stages;     // multiple of kConsumerWarps: stage s belongs to warp s % kConsumerWarps
  int stage_bytes;
  int vec_floats;   // shared vector buffer, including the norm-gain buffer at gbuf_off
  int gbuf_off;     // float offset of the fp16 norm-gain buffer inside the vector buffer
  int rslice_off;   // MoE: float offset of the fp16 router slice [E][own rows] inside the vector buffer
  int rslice_rows;  // MoE: own-row capacity of each expert's slice
  int xplane;       // float offset of the second-half plane of the input vector (see Consumer::xv)
};

}  // namespace kie
