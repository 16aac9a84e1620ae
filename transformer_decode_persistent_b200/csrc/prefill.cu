// Chunked prompt prefill for dense models on B200 (sm_100a) tensor cores.
//
// Before the first decode step the engine must hold the KV cache of every
// prompt position. The pages' persistent kernel covers the per-token decode
// step ("メモリの壁を打破する：標準的なGPUで3,000 tokens/sの推論を実現する", section
// "1. The Monokernel Runtime"); a long prompt is a different workload that the
// pages leave open ("Kog、より深いGPU最適化でAI推論を高速化できると賭ける", section
// "Kogのベンチマークでは決着しないこと": long prompts and contexts are the untested
// case). Processed as chunks of up to kChunk tokens, the prompt's projections
// are dense contractions, so they run on the 5th-generation tensor cores:
//
//  * gemm_kernel: D[128 weight rows x 128 tokens] = W[rows, K] . X[tokens, K]^T
//    with tcgen05.mma (kind::f16, fp32 accumulator in tensor memory). TMA
//    loads 64-wide K slices of W and X with 128-byte swizzle into a 4-stage
//    shared-memory ring; one thread issues the MMAs, another the loads, and
//    four warps read the accumulator back with tcgen05.ld for a fused
//    epilogue. The activations enter as two fp16 parts, hi = fp16(x) and
//    lo = fp16(x - hi), accumulated into the same fp32 accumulator, so the
//    products carry about 22 bits of the fp32 activation (a single fp16
//    operand would carry 11); the weights are fp16 already.
//  * epilogues: q/k/v (RoPE on adjacent row pairs, q scaled by 1/sqrt(dh), K
//    and V appended to the fp16 cache the decode kernel reads), residual add
//    (output and down projections) and SwiGLU (gate/up rows interleaved).
//  * rmsnorm_split_kernel, embed_kernel and tc_attention_kernel (causal softmax
//    attention of the chunk over the cache on the tensor cores, mma.sync with
//    fp16 operands (q as hi/lo parts) and fp32 accumulators).
//
// The last layer's attention, output projection and FFN are skipped: a
// prompt position contributes nothing but its K and V.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "prefill.h"

namespace kie {
namespace pf {

// ---------------------------------------------------------------- GEMM

constexpr int kStageBytes = kTileA + 2 * kTileB;
constexpr unsigned kSpinLimit = 1u << 28;  // bounded mbarrier waits (several seconds)

__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool mbar_try(uint32_t b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(b), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; on giving up it records an error and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t b, unsigned parity, int* err) {
  for (unsigned i = 0; i < kSpinLimit; ++i)
    if (mbar_try(b, parity)) return true;
  atomicExch(err, 1);
  return false;
}

// K-major operand tile in shared memory as TMA writes it with 128-byte
// swizzle: rows of 64 fp16 (128 bytes), 8-row groups 1024 bytes apart. The
// descriptor fields: start address >> 4 (bits 0-13), leading byte offset 1
// (unused by swizzled K-major layouts), stride byte offset 1024 >> 4 (bits
// 32-45), descriptor version 1 (bits 46-47), swizzle mode 128B = 2 (bits
// 61-63). A K step of 16 elements advances the start address by 32 bytes.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and
// B fp16 (formats 0), both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mma(uint32_t tmem, uint64_t a, uint64_t b, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"((unsigned)acc)
      : "memory");
}
__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

__device__ __forceinline__ void split_store(__half* hi, __half* lo, size_t i, float v) {
  const __half h = __float2half_rn(v);
  hi[i] = h;
  lo[i] = __float2half_rn(v - __half2float(h));
}

// Epilogue for one 32-token slice of the accumulator: this thread holds
// D[row][n .. n+32) (row = this thread's weight row). Rows beyond M and
// tokens beyond N are skipped; the lane-pair exchanges run on every lane. tb
// is the first token row of a device-resident range (0 otherwise): output
// rows are tb + n + j.
__device__ __forceinline__ void epilogue(const GemmArgs& a, int row, int tb, int n, int N, const float (&v)[32]) {
  const int lane = threadIdx.x & 31;
  const bool row_ok = row < a.M;
  if (a.epi == EPI_RESID) {
    if (!row_ok) return;
#pragma unroll 4
    for (int j = 0; j < 32; ++j)
      if (n + j < N) a.x[(size_t)(tb + n + j) * a.M + row] += v[j];
    return;
  }
  if (a.epi == EPI_STORE) {
    if (!row_ok) return;
#pragma unroll 4
    for (int j = 0; j < 32; ++j)
      if (n + j < N) a.out[(size_t)(tb + n + j) * a.M + row] = v[j];
    return;
  }
  if (a.epi == EPI_SWIGLU) {
    // rows 2j (gate) and 2j+1 (up) sit on lanes 2i and 2i+1 of one warp
#pragma unroll 4
    for (int j = 0; j < 32; ++j) {
      const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
      if (row_ok && !(lane & 1) && n + j < N) {
        const float h = silu(v[j]) * other;
        split_store(a.h_hi, a.h_lo, (size_t)(tb + n + j) * a.ff + row / 2, h);
      }
    }
    return;
  }
  // EPI_QKV: virtual rows of a head run dims 0, dh/2, 1, dh/2 + 1, ... so a
  // RoPE pair (i, i + dh/2) sits on lanes 2p and 2p+1
  const int dh = a.dh, H = row / dh, vr = row - H * dh, pi = vr >> 1;
  const int dim = (vr & 1) ? pi + dh / 2 : pi;
  const float scale = rsqrtf((float)dh);
#pragma unroll 2
  for (int j = 0; j < 32; ++j) {
    const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
    const int t = n + j;
    if (!row_ok || t >= N) continue;
    const int pos = a.pos0 + t;
    if (H < a.hq + a.hk) {
      const float2 cs = a.rope[(size_t)pos * (dh / 2) + pi];
      const float x0 = (vr & 1) ? other : v[j], x1 = (vr & 1) ? v[j] : other;
      const float r = (vr & 1) ? (x0 * cs.y + x1 * cs.x) : (x0 * cs.x - x1 * cs.y);
      if (H < a.hq) {
        a.q[(size_t)t * a.hq * dh + (size_t)H * dh + dim] = r * scale;
      } else {
        a.kcache[((size_t)(a.layer * a.hk + (H - a.hq)) * a.max_ctx + pos) * dh + dim] = __float2half_rn(r);
      }
    } else {
      a.vcache[((size_t)(a.layer * a.hk + (H - a.hq - a.hk)) * a.max_ctx + pos) * dh + dim] = __float2half_rn(v[j]);
    }
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBh,
                const __grid_constant__ CUtensorMap tmBl, const GemmArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint32_t* taddr_s = reinterpret_cast<uint32_t*>(accf + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // token tiles vary fastest: the CTAs that share a weight tile run together
  // and read it through L2 (measured 1.5 % faster on a 32K prompt)
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
  const int nkb = (a.K + kBK - 1) / kBK;
  // tokens: B rows tb .. tb + N - 1 (a device-resident range, or 0 .. a.N - 1)
  int tb = 0, N = a.N;
  if (a.nrange) {
    tb = a.nrange[0];
    N = min(a.N, a.nrange[1]);
  }
  if (n0 >= N) return;  // the whole CTA: before any barrier or tensor-memory allocation
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&full[s])));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&empty[s])));
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(accf)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(taddr_s)),
                 "r"(kBN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *taddr_s;
  bool ok = true;

  if (warp == 0 && lane == 0) {
    // TMA producer
    int issued = 0;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int s = kb % kStages;
      const unsigned r = (unsigned)(kb / kStages);
      if (r > 0) ok = mbar_wait(su32(&empty[s]), (r - 1) & 1u, a.err);
      if (!ok) break;
      ++issued;
      unsigned char* st = smem + s * kStageBytes;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(&full[s])), "r"(kStageBytes)
                   : "memory");
      tma2d(su32(st), &tmA, kb * kBK, m0, su32(&full[s]));
      tma2d(su32(st + kTileA), &tmBh, kb * kBK, tb + n0, su32(&full[s]));
      tma2d(su32(st + kTileA + kTileB), &tmBl, kb * kBK, tb + n0, su32(&full[s]));
    }
    // let every copy this thread issued land before the CTA can exit (on the
    // normal path the MMA issuer has already waited for all of them)
    for (int kb = issued - 1; kb >= 0 && kb >= issued - kStages; --kb)
      mbar_wait(su32(&full[kb % kStages]), (unsigned)(kb / kStages) & 1u, a.err);
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int s = kb % kStages;
      ok = mbar_wait(su32(&full[s]), (unsigned)(kb / kStages) & 1u, a.err);
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = su32(smem + s * kStageBytes);
      const uint64_t da = sdesc(sa), dhi = sdesc(sa + kTileA), dlo = sdesc(sa + kTileA + kTileB);
#pragma unroll
      for (int ks = 0; ks < kBK / 16; ++ks) {
        mma(tmem, da + 2 * ks, dhi + 2 * ks, kb > 0 || ks > 0);
        mma(tmem, da + 2 * ks, dlo + 2 * ks, true);
      }
      commit(su32(&empty[s]));  // the stage is free once these MMAs have read it
    }
    commit(su32(accf));  // arrives once every MMA issued above has completed
  }
  __syncwarp();

  // epilogue: warp w reads accumulator lanes (rows) 32w .. 32w + 31
  ok = mbar_wait(su32(accf), 0u, a.err);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  // tcgen05.ld is warp-collective: the warp reads the accumulator only if every
  // lane's wait succeeded (a failed wait has already flagged the error)
  if (__all_sync(0xffffffffu, ok)) {
    const int row = m0 + warp * 32 + lane;
    for (int c = 0; c < kBN; c += 32) {
      float v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      if (n0 + c < N) epilogue(a, row, tb, n0 + c, N, v);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kBN));
}

// ---------------------------------------------------------------- small kernels

// x[t] = E[tok[t]] (fp16 -> fp32), one block per token
__global__ void embed_kernel(const int* tok, const __half* E, float* x, int d) {
  const int t = blockIdx.x;
  const __half* e = E + (size_t)tok[t] * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) x[(size_t)t * d + i] = __half2float(e[i]);
}

// xn = x / sqrt(mean(x^2) + eps) * g, written as fp16 hi and lo parts; one
// block of 256 threads per token
__global__ void rmsnorm_split_kernel(const float* x, const __half* g, __half* hi, __half* lo, int d, float eps) {
  __shared__ float red[8];
  const int t = blockIdx.x;
  const float* xr = x + (size_t)t * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) ss = fmaf(xr[i], xr[i], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
  const float inv = 1.0f / sqrtf(tot / (float)d + eps);
  for (int i = threadIdx.x; i < d; i += blockDim.x) split_store(hi, lo, (size_t)t * d + i, xr[i] * inv * __half2float(g[i]));
}

// ---------------------------------------------------------------- MoE routing

constexpr int kRouteThreads = 1024;
constexpr int kRoutePerLane = 8;  // experts a lane holds: up to 256 experts

// One block for the whole chunk. (1) Warp w routes tokens w, w + 32, ...: the
// softmax numerators of the token's router logits (the denominator cancels in
// the renormalisation), top_k rounds of a warp arg-max with the lower expert
// index on ties, weights renormalised over the chosen. (2) Warp w counts and
// ranks the (token, slot) pairs of experts w, w + 32, ... in pair order
// (ballots), so the sorted order is the pair order within each expert. (3)
// Offsets and each pair's row in the expert-sorted order.
__global__ void __launch_bounds__(kRouteThreads) moe_route_kernel(RouteArgs a) {
  extern __shared__ int sm_route[];
  int* rank = sm_route;                     // [T * top_k]
  int* off = rank + a.T * a.top_k;          // [E]
  int* cnt = off + a.E;                     // [E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = kRouteThreads / 32;
  const int P = a.T * a.top_k;
  for (int t = warp; t < a.T; t += nw) {
    const float* lg = a.logits + (size_t)t * a.E;
    float pr[kRoutePerLane];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kRoutePerLane; ++i) {
      const int e = lane + 32 * i;
      pr[i] = e < a.E ? lg[e] : -INFINITY;
      mx = fmaxf(mx, pr[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
#pragma unroll
    for (int i = 0; i < kRoutePerLane; ++i) pr[i] = (lane + 32 * i < a.E) ? expf(pr[i] - mx) : -1.f;
    float wsum = 0.f;
    for (int k = 0; k < a.top_k; ++k) {
      float bv = -1.f;
      int bi = INT_MAX;
#pragma unroll
      for (int i = 0; i < kRoutePerLane; ++i)
        if (pr[i] > bv) {
          bv = pr[i];
          bi = lane + 32 * i;
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (bi >= a.E) {  // a non-finite logit: flag it and keep the index valid
        if (lane == 0) atomicExch(a.err, 2);
        bi = k;
        bv = 0.f;
      }
#pragma unroll
      for (int i = 0; i < kRoutePerLane; ++i)
        if (lane + 32 * i == bi) pr[i] = -1.f;
      if (lane == 0) {
        a.sel[t * a.top_k + k] = bi;
        a.wt[t * a.top_k + k] = bv;
      }
      wsum += bv;
    }
    __syncwarp();
    if (lane < a.top_k) a.wt[t * a.top_k + lane] = wsum > 0.f ? a.wt[t * a.top_k + lane] / wsum : 0.f;
  }
  __syncthreads();
  for (int e = warp; e < a.E; e += nw) {
    int run = 0;
    for (int i0 = 0; i0 < P; i0 += 32) {
      const int i = i0 + lane;
      const bool m = i < P && a.sel[i] == e;
      const unsigned b = __ballot_sync(0xffffffffu, m);
      if (m) rank[i] = run + __popc(b & ((1u << lane) - 1u));
      run += __popc(b);
    }
    if (lane == 0) cnt[e] = run;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int o = 0;
    for (int e = 0; e < a.E; ++e) {
      off[e] = o;
      a.range[2 * e] = o;
      a.range[2 * e + 1] = cnt[e];
      o += cnt[e];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < P; i += kRouteThreads) {
    const int row = off[a.sel[i]] + rank[i];
    a.row_of[i] = row;
    a.tok_of[row] = i / a.top_k;
  }
}

// ghi/glo[r] = hi/lo[tok_of[r]] (rows of d fp16), one block per row
__global__ void moe_gather_kernel(const int* tok_of, const __half* hi, const __half* lo, __half* ghi, __half* glo,
                                  int d) {
  const int r = blockIdx.x;
  const size_t src = (size_t)tok_of[r] * d, dst = (size_t)r * d;
  for (int i = threadIdx.x * 8; i < d; i += blockDim.x * 8) {
    *reinterpret_cast<uint4*>(ghi + dst + i) = *reinterpret_cast<const uint4*>(hi + src + i);
    *reinterpret_cast<uint4*>(glo + dst + i) = *reinterpret_cast<const uint4*>(lo + src + i);
  }
}

// x[t] += sum_k wt[t][k] * y[row_of[t][k]], k in order; one block per token
__global__ void moe_combine_kernel(const float* y, const int* row_of, const float* wt, float* x, int top_k, int d) {
  const int t = blockIdx.x;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float acc = 0.f;
    for (int k = 0; k < top_k; ++k) acc = fmaf(wt[t * top_k + k], y[(size_t)row_of[t * top_k + k] * d + i], acc);
    x[(size_t)t * d + i] += acc;
  }
}

// ---------------------------------------------------------------- tensor-core attention
//
// Causal attention of the chunk's queries on the tensor cores (mma.sync
// m16n8k16, fp16 operands, fp32 accumulators): block (query head h, 64
// queries), 4 warps of 16 query rows. q (fp32, rotated, pre-scaled) enters as
// fp16 hi + lo parts held in registers; K and V blocks of 64 keys stream
// through double-buffered, padded shared memory (cp.async). S = Q_hi K^T +
// Q_lo K^T keeps about 22 bits of q (score errors are amplified by the
// exponential); the online softmax runs on the accumulators; P (in [0, 1]) is
// rounded once to fp16 for O += P V, a relative error of at most 2^-11 per
// weight, below the fp16 rounding of V itself. Output as fp16 hi/lo parts
// [T][hq * dh] (the next GEMM's operand).
constexpr int kTQ = 64, kTK = 64;
template <int DH>
struct TcAttn {
  static constexpr int LD = DH + 8;  // padded row (halves): ldmatrix rows fall in distinct banks
  static constexpr int kTileHalves = kTK * LD;
  static constexpr int kSmem = 2 * 2 * kTileHalves * 2;  // K and V, double-buffered
};

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}
__device__ __forceinline__ void split_h2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half ha = __float2half_rn(a), hb = __float2half_rn(b);
  const __half2 h = __halves2half2(ha, hb);
  memcpy(&hi, &h, 4);
  lo = pack_h2(a - __half2float(ha), b - __half2float(hb));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <int DH>
__global__ void __launch_bounds__(128) tc_attention_kernel(AttnArgs a) {
  using C = TcAttn<DH>;
  constexpr int NKS = DH / 16;  // k-steps of q . k
  constexpr int NDT = DH / 8;   // n-tiles of the output
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __half* sK = reinterpret_cast<__half*>(smem_raw);  // [2][kTK][LD]
  __half* sV = sK + 2 * C::kTileHalves;               // [2][kTK][LD]
  const int h = blockIdx.x, qb = blockIdx.y;
  const int g = (h * a.hk) / a.hq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int t0 = qb * kTQ;                      // first query (chunk index) of the block
  const int rw = t0 + warp * 16;                // first query row of this warp
  const int qlast = min(a.T, t0 + kTQ) - 1;     // last query of the block
  const int last = a.pos0 + qlast;              // last key any query of the block sees
  const __half* K = a.kcache + (size_t)(a.layer * a.hk + g) * a.max_ctx * DH;
  const __half* V = a.vcache + (size_t)(a.layer * a.hk + g) * a.max_ctx * DH;

  // q fragments (A operand, row-major 16 x 16 per k-step) as hi and lo parts
  uint32_t qh[NKS][4], ql[NKS][4];
  {
    const int r0 = rw + gid, r1 = rw + gid + 8;
    const float* q0 = a.q + (size_t)r0 * a.hq * DH + (size_t)h * DH;
    const float* q1 = a.q + (size_t)r1 * a.hq * DH + (size_t)h * DH;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
      const int c = ks * 16 + tig * 2;
      float2 x00 = make_float2(0.f, 0.f), x10 = x00, x01 = x00, x11 = x00;
      if (r0 < a.T) { x00 = *reinterpret_cast<const float2*>(q0 + c); x01 = *reinterpret_cast<const float2*>(q0 + c + 8); }
      if (r1 < a.T) { x10 = *reinterpret_cast<const float2*>(q1 + c); x11 = *reinterpret_cast<const float2*>(q1 + c + 8); }
      split_h2(x00.x, x00.y, qh[ks][0], ql[ks][0]);
      split_h2(x10.x, x10.y, qh[ks][1], ql[ks][1]);
      split_h2(x01.x, x01.y, qh[ks][2], ql[ks][2]);
      split_h2(x11.x, x11.y, qh[ks][3], ql[ks][3]);
    }
  }
  float o[NDT][4];
#pragma unroll
  for (int i = 0; i < NDT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows gid and gid + 8
  const int pos_r0 = a.pos0 + rw + gid, pos_r1 = pos_r0 + 8;

  // K/V block loader: 64 rows x DH halves each, 16-byte cp.async pieces
  auto load_kv = [&](int buf, int j0) {
    constexpr int PIECES = kTK * DH / 8;
    __half* dk = sK + buf * C::kTileHalves;
    __half* dv = sV + buf * C::kTileHalves;
    for (int i = threadIdx.x; i < PIECES; i += 128) {
      const int r = i / (DH / 8), c = (i - r * (DH / 8)) * 8;
      const int key = min(j0 + r, last);  // rows past `last` repeat a valid row (masked below)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(su32(dk + r * C::LD + c)),
                   "l"(K + (size_t)key * DH + c)
                   : "memory");
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(su32(dv + r * C::LD + c)),
                   "l"(V + (size_t)key * DH + c)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  const int nkb = last / kTK + 1;
  load_kv(0, 0);
  for (int kb = 0; kb < nkb; ++kb) {
    const int buf = kb & 1;
    if (kb + 1 < nkb) {
      load_kv(buf ^ 1, (kb + 1) * kTK);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const int j0 = kb * kTK;
    const __half* cK = sK + buf * C::kTileHalves;
    const __half* cV = sV + buf * C::kTileHalves;
    // S = Q K^T for 16 rows x 64 keys: 8 n-tiles of 8 keys
    float s[kTK / 8][4];
#pragma unroll
    for (int nt = 0; nt < kTK / 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
#pragma unroll
      for (int np = 0; np < kTK / 16; ++np) {
        // B fragments of two n-tiles (keys 16np .. 16np + 15) for dims 16ks .. 16ks + 15:
        // matrices (keys +0..7, dims +0..7), (+0..7, +8..15), (+8..15, +0..7), (+8..15, +8..15)
        const int mi = lane >> 3, mr = lane & 7;
        const int key = np * 16 + (mi >> 1) * 8 + mr, dim = ks * 16 + (mi & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(su32(cK + key * C::LD + dim), b0, b1, b2, b3);
        mma16816(s[2 * np], qh[ks], b0, b1);
        mma16816(s[2 * np], ql[ks], b0, b1);
        mma16816(s[2 * np + 1], qh[ks], b2, b3);
        mma16816(s[2 * np + 1], ql[ks], b2, b3);
      }
    }
    // causal mask and online softmax (rows gid, gid + 8; each row over the quad)
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int nt = 0; nt < kTK / 8; ++nt) {
      const int k0 = j0 + nt * 8 + tig * 2;
      if (k0 > pos_r0) s[nt][0] = -INFINITY;
      if (k0 + 1 > pos_r0) s[nt][1] = -INFINITY;
      if (k0 > pos_r1) s[nt][2] = -INFINITY;
      if (k0 + 1 > pos_r1) s[nt][3] = -INFINITY;
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
    }
    const float c0 = (mx0 == -INFINITY) ? 1.f : expf(m0 - mx0);
    const float c1 = (mx1 == -INFINITY) ? 1.f : expf(m1 - mx1);
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < kTK / 8; ++nt) {
      s[nt][0] = (s[nt][0] == -INFINITY) ? 0.f : expf(s[nt][0] - mx0);
      s[nt][1] = (s[nt][1] == -INFINITY) ? 0.f : expf(s[nt][1] - mx0);
      s[nt][2] = (s[nt][2] == -INFINITY) ? 0.f : expf(s[nt][2] - mx1);
      s[nt][3] = (s[nt][3] == -INFINITY) ? 0.f : expf(s[nt][3] - mx1);
      ps0 += s[nt][0] + s[nt][1];
      ps1 += s[nt][2] + s[nt][3];
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      ps0 += __shfl_xor_sync(0xffffffffu, ps0, o2);
      ps1 += __shfl_xor_sync(0xffffffffu, ps1, o2);
    }
    l0 = l0 * c0 + ps0;
    l1 = l1 * c1 + ps1;
    m0 = mx0;
    m1 = mx1;
#pragma unroll
    for (int i = 0; i < NDT; ++i) {
      o[i][0] *= c0;
      o[i][1] *= c0;
      o[i][2] *= c1;
      o[i][3] *= c1;
    }
    // O += P V: P from the S accumulators (A layout), V via transposed ldmatrix
#pragma unroll
    for (int kk = 0; kk < kTK / 16; ++kk) {
      uint32_t ph[4];
      ph[0] = pack_h2(s[2 * kk][0], s[2 * kk][1]);
      ph[1] = pack_h2(s[2 * kk][2], s[2 * kk][3]);
      ph[2] = pack_h2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      ph[3] = pack_h2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < NDT / 2; ++dp) {
        // B fragments of two dim n-tiles (dims 16dp .. 16dp + 15) for keys 16kk .. 16kk + 15:
        // transposed matrices (keys +0..7, dims +0..7), (+8..15, +0..7), (+0..7, +8..15), (+8..15, +8..15)
        const int mi = lane >> 3, mr = lane & 7;
        const int key = kk * 16 + (mi & 1) * 8 + mr, dim = dp * 16 + (mi >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(su32(cV + key * C::LD + dim), b0, b1, b2, b3);
        mma16816(o[2 * dp], ph, b0, b1);
        mma16816(o[2 * dp + 1], ph, b2, b3);
      }
    }
    __syncthreads();  // this buffer is reloaded two blocks on
  }
  // O / l to the fp16 hi/lo output
  const int r0 = rw + gid, r1 = r0 + 8;
  const float i0 = 1.0f / l0, i1 = 1.0f / l1;
#pragma unroll
  for (int nt = 0; nt < NDT; ++nt) {
    const int c = nt * 8 + tig * 2;
    if (r0 < a.T) {
      const size_t at = (size_t)r0 * a.hq * DH + (size_t)h * DH + c;
      split_store(a.o_hi, a.o_lo, at, o[nt][0] * i0);
      split_store(a.o_hi, a.o_lo, at + 1, o[nt][1] * i0);
    }
    if (r1 < a.T) {
      const size_t at = (size_t)r1 * a.hq * DH + (size_t)h * DH + c;
      split_store(a.o_hi, a.o_lo, at, o[nt][2] * i1);
      split_store(a.o_hi, a.o_lo, at + 1, o[nt][3] * i1);
    }
  }
}

// ---------------------------------------------------------------- host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

}  // namespace

bool make_map(CUtensorMap* map, const __half* base, int rows, int cols, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t gemm(const CUtensorMap& A, const CUtensorMap& Bh, const CUtensorMap& Bl, const GemmArgs& a,
                 cudaStream_t st) {
  // the shared-memory opt-in is per device; setting it again is harmless
  static bool attr[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr[dev] = true;
  }
  const dim3 grid((a.N + kBN - 1) / kBN, (a.M + kBM - 1) / kBM);
  gemm_kernel<<<grid, kGemmThreads, kGemmSmem, st>>>(A, Bh, Bl, a);
  return cudaGetLastError();
}

cudaError_t embed(const int* tok, const __half* E, float* x, int T, int d, cudaStream_t st) {
  embed_kernel<<<T, 256, 0, st>>>(tok, E, x, d);
  return cudaGetLastError();
}

cudaError_t rmsnorm_split(const float* x, const __half* g, __half* hi, __half* lo, int T, int d, float eps,
                          cudaStream_t st) {
  rmsnorm_split_kernel<<<T, 256, 0, st>>>(x, g, hi, lo, d, eps);
  return cudaGetLastError();
}

cudaError_t moe_route(const RouteArgs& a, cudaStream_t st) {
  const int smem = (a.T * a.top_k + 2 * a.E) * 4;
  static bool attr[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(moe_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (kChunk * 8 + 2 * 256) * 4);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr[dev] = true;
  }
  moe_route_kernel<<<1, kRouteThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t moe_gather(const int* tok_of, const __half* hi, const __half* lo, __half* ghi, __half* glo, int rows,
                       int d, cudaStream_t st) {
  moe_gather_kernel<<<rows, 128, 0, st>>>(tok_of, hi, lo, ghi, glo, d);
  return cudaGetLastError();
}

cudaError_t moe_combine(const float* y, const int* row_of, const float* wt, float* x, int T, int top_k, int d,
                        cudaStream_t st) {
  moe_combine_kernel<<<T, 256, 0, st>>>(y, row_of, wt, x, top_k, d);
  return cudaGetLastError();
}

cudaError_t attention(const AttnArgs& a, cudaStream_t st) {
  const dim3 grid(a.hq, (a.T + kTQ - 1) / kTQ);
  static bool attr[64][2] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const int k = a.dh == 128 ? 1 : 0;
  if (dev < 0 || dev >= 64 || !attr[dev][k]) {
    cudaError_t e = k ? cudaFuncSetAttribute(tc_attention_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             TcAttn<128>::kSmem)
                      : cudaFuncSetAttribute(tc_attention_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             TcAttn<64>::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr[dev][k] = true;
  }
  if (k) tc_attention_kernel<128><<<grid, 128, TcAttn<128>::kSmem, st>>>(a);
  else tc_attention_kernel<64><<<grid, 128, TcAttn<64>::kSmem, st>>>(a);
  return cudaGetLastError();
}


}  // namespace pf
}  // namespace kie
