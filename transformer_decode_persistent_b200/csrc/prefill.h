// Chunked tensor-core prompt prefill (dense and MoE models): kernels and
// launchers of prefill.cu, used by the host side of libkie. Internal, not part
// of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace kie {
namespace pf {

constexpr int kBM = 128;  // weight rows per GEMM tile (accumulator lanes)
constexpr int kBN = 128;  // tokens per GEMM tile (accumulator columns)
constexpr int kBK = 64;   // K elements per pipeline stage (one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr int kTileA = kBM * kBK * 2;
constexpr int kTileB = kBN * kBK * 2;
constexpr int kGemmThreads = 128;
constexpr int kGemmSmem = kStages * (kTileA + 2 * kTileB) + 1024 + 256;
constexpr int kChunk = 1024;  // prompt tokens per chunk (activation buffers hold this many)

enum Epi { EPI_QKV = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_STORE = 3 };

struct GemmArgs {
  int M, N, K;  // weight rows, tokens, input length
  int epi;
  // EPI_QKV: rows in the packed q/k/v order (head dims 0, dh/2, 1, dh/2+1, ...)
  float* q;                  // [N][hq * dh] rotated q, scaled by 1/sqrt(dh)
  __half *kcache, *vcache;   // [L][hk][max_ctx][dh]
  const float2* rope;        // [max_ctx][dh/2] (cos, sin)
  int layer, hq, hk, dh, max_ctx, pos0;
  // EPI_RESID: x[N][M] += D^T
  float* x;
  // EPI_SWIGLU: rows gate_0, up_0, gate_1, ...; h[N][ff] = silu(gate) * up as fp16 hi/lo
  __half *h_hi, *h_lo;
  int ff;
  // EPI_STORE: out[N][M] = D^T (fp32)
  float* out;
  // token rows taken from a device-resident range (one routed expert's rows
  // of the expert-sorted activations): when nrange is set, the tokens are rows
  // nrange[0] .. nrange[0] + nrange[1] - 1 of B and of the output (N is then
  // only the grid's bound); tiles past the count exit at once
  const int* nrange;
  int* err;  // set to 1 when a bounded wait gives up
};

// MoE routing of a chunk (the decode kernel's rule): per token, softmax
// numerators of the router logits, the top_k by value with the lower expert
// index on ties, weights renormalised over the chosen ones.
struct RouteArgs {
  const float* logits;  // [T][E]
  int* sel;             // [T][top_k] chosen experts
  float* wt;            // [T][top_k] their weights
  int* range;           // [E][2]: row offset and count of each expert in the sorted pairs
  int* row_of;          // [T][top_k]: the pair's row in the expert-sorted order
  int* tok_of;          // [T * top_k]: the token of each sorted row
  int* err;             // set to 2 on a non-finite router logit
  int T, E, top_k;
};

struct AttnArgs {
  const float* q;  // [T][hq * dh]
  const __half *kcache, *vcache;
  __half *o_hi, *o_lo;  // [T][hq * dh]
  int T, pos0, layer, hq, hk, dh, max_ctx;
};

// 2-D fp16 tensor map [rows][cols] (row-major) with boxes of kBK columns x
// box_rows rows and 128-byte swizzle; false if the encoder is unavailable or
// rejects the shape.
bool make_map(CUtensorMap* map, const __half* base, int rows, int cols, int box_rows);
cudaError_t gemm(const CUtensorMap& A, const CUtensorMap& Bh, const CUtensorMap& Bl, const GemmArgs& a,
                 cudaStream_t st);
cudaError_t embed(const int* tok, const __half* E, float* x, int T, int d, cudaStream_t st);
cudaError_t rmsnorm_split(const float* x, const __half* g, __half* hi, __half* lo, int T, int d, float eps,
                          cudaStream_t st);
// causal attention of a chunk over the cache on the tensor cores (mma.sync)
cudaError_t attention(const AttnArgs& a, cudaStream_t st);
// MoE: routing, the stable sort of (token, slot) pairs by expert, the gather of
// the normalised rows in that order, and the weighted combine of the experts'
// outputs into the residual stream (x[t] += sum_k wt[t][k] y[row_of[t][k]], k
// in order)
cudaError_t moe_route(const RouteArgs& a, cudaStream_t st);
cudaError_t moe_gather(const int* tok_of, const __half* hi, const __half* lo, __half* ghi, __half* glo, int rows,
                       int d, cudaStream_t st);
cudaError_t moe_combine(const float* y, const int* row_of, const float* wt, float* x, int T, int top_k, int d,
                        cudaStream_t st);

}  // namespace pf
}  // namespace kie
