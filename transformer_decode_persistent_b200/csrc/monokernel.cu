// Persistent batch-1 decode kernel for B200 (sm_100a).
//
// One cooperative launch runs n whole decode steps: "MatMul, attention,
// normalization and sampling" inside one GPU-resident program that feeds each
// new token back to itself without returning to the host ("メモリの壁を打破する：
// 標準的なGPUで3,000 tokens/sの推論を実現する", section "1. The Monokernel Runtime").
// At batch 1 the step is bound by moving every active weight from HBM once per
// token (same page, section "ボトルネック：計算量ではなくメモリ帯域幅"), so the
// kernel is organised around keeping HBM busy:
//
//  * One CTA per SM. Each CTA owns a contiguous region of a packed "weight
//    tape" that holds, in execution order, its slice of every matrix of one
//    decode step (see kie_internal.h for the tile format).
//  * Warp 8 of each CTA is a producer: one lane streams the CTA's tape into a
//    ring of shared-memory stages with TMA bulk copies (cp.async.bulk, L2
//    evict-first), completion tracked by mbarriers. It never waits for the
//    grid barriers, so the next phase's (and next layer's) weights are already
//    in flight while the current phase reduces and synchronises.
//  * Warps 0-7 are consumers: GEMV on each tile against the fp32 input vector
//    held in shared memory (fp16 weights, fp32 FMA), RMSNorm (recomputed by
//    every CTA from the L2-resident residual), RoPE, split-K attention over the
//    fp16 KV cache, SwiGLU, residual adds, the LM head and a greedy argmax.
//  * Dependent phases are joined by a grid barrier (monotonic arrival counter,
//    release/acquire at GPU scope) with a %globaltimer deadline: the
//    synchronisation cost the pages name ("マイクロ秒が失われる場所") is paid in a
//    few hundred ns, and hidden behind the producer's prefetch.
//
// Every wait (grid barrier, ring stages, routing hand-off) is bounded: on a
// deadline the kernel records KIE_ERR_TIMEOUT in the control block, raises an
// abort flag that all CTAs poll, lets in-flight bulk copies land, and returns.
#include <cuda_fp16.h>
#include <float.h>
#include <limits.h>
#include <stdint.h>

#include "kie_internal.h"

namespace kie {

constexpr int kMaxStages = 16;
constexpr int kErrTimeout = -5;  // KIE_ERR_TIMEOUT
constexpr int kErrDevice = -6;   // KIE_ERR_DEVICE

struct SmemCtl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t route_bar;
  volatile int abort;
  int tok;
  float margin;
  int route_e[kMaxTopK];
  float route_w[kMaxTopK];
  float red[64];
  Cand wcand[kConsumerWarps];
};

// Shared-memory layout, identical on host and device.
__host__ __device__ inline int smem_ctl_bytes() { return (int)((sizeof(SmemCtl) + 127) & ~127); }
__host__ __device__ inline int smem_ring_offset(int vec_floats) {
  int b = smem_ctl_bytes() + kPartFloats * 4 + vec_floats * 4;
  return (b + 1023) & ~1023;
}
__host__ __device__ inline int smem_total(int vec_floats, int n_stages) {
  return smem_ring_offset(vec_floats) + n_stages * kStageBytes;
}

// ---------------------------------------------------------------- primitives

__device__ __forceinline__ uint32_t su32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, unsigned n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar,
                                         unsigned long long policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(su32(dst)),
      "l"(src), "r"(bytes), "r"(su32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// consumer-only barrier (named barrier 1 over the 256 consumer threads)
__device__ __forceinline__ void cbar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// 8 fp16 weights (one 16-byte chunk) against 8 fp32 inputs, accumulated in fp32.
__device__ __forceinline__ float dot8(const uint4& w, const float4& a, const float4& b, float acc) {
  const __half2* h = reinterpret_cast<const __half2*>(&w);
  float2 f0 = __half22float2(h[0]);
  float2 f1 = __half22float2(h[1]);
  float2 f2 = __half22float2(h[2]);
  float2 f3 = __half22float2(h[3]);
  acc = fmaf(f0.x, a.x, acc);
  acc = fmaf(f0.y, a.y, acc);
  acc = fmaf(f1.x, a.z, acc);
  acc = fmaf(f1.y, a.w, acc);
  acc = fmaf(f2.x, b.x, acc);
  acc = fmaf(f2.y, b.y, acc);
  acc = fmaf(f3.x, b.z, acc);
  acc = fmaf(f3.y, b.w, acc);
  return acc;
}

// Greedy candidate merge: largest value, lowest index on ties, and the
// second-largest value of the union (equal to the first on a tie).
__device__ __forceinline__ void cand_merge(float& v1, int& i1, float& v2, float b1, int bi, float b2) {
  if (b1 > v1 || (b1 == v1 && bi < i1)) {
    v2 = fmaxf(v1, b2);
    v1 = b1;
    i1 = bi;
  } else {
    v2 = fmaxf(v2, b1);
  }
}
__device__ __forceinline__ void cand_warp_merge(float& v1, int& i1, float& v2) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float b1 = __shfl_xor_sync(0xffffffffu, v1, o);
    int bi = __shfl_xor_sync(0xffffffffu, i1, o);
    float b2 = __shfl_xor_sync(0xffffffffu, v2, o);
    cand_merge(v1, i1, v2, b1, bi, b2);
  }
}

// ---------------------------------------------------------------- errors

__device__ void record_error(const Params& P, int code, int where, int step) {
  if (atomicCAS(&P.ctrl->err, 0, code) == 0) {
    P.ctrl->err_cta = blockIdx.x;
    P.ctrl->err_step = step;
    P.ctrl->err_where = where;
  }
  __threadfence();
  atomicExch(&P.ctrl->abort, 1u);
}

// Bounded wait on an mbarrier phase. Returns false on abort or deadline.
__device__ bool wait_bar(const Params& P, SmemCtl* sc, uint64_t* b, unsigned parity, int where,
                         int step) {
  if (mbar_test(b, parity)) return true;
  const unsigned long long t0 = gtimer();
  for (unsigned it = 1;; ++it) {
    if (mbar_test(b, parity)) return true;
    if ((it & 7) == 0) {
      if (sc->abort || ld_relaxed(&P.ctrl->abort)) {
        sc->abort = 1;
        return false;
      }
      if (gtimer() - t0 > P.timeout_ns) {
        record_error(P, kErrTimeout, where, step);
        sc->abort = 1;
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------- producer

struct Producer {
  const Params& P;
  SmemCtl* sc;
  unsigned char* ring;
  unsigned long long pol;
  unsigned t = 0;  // tiles issued
  int step = 0;

  __device__ Producer(const Params& p, SmemCtl* s, unsigned char* r) : P(p), sc(s), ring(r) {
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  }

  __device__ bool issue(const SegDesc& sd, const SegShape& sh) {
    const int ngroups = (sd.nrows + sh.g - 1) / sh.g;
    const unsigned char* base = P.tape + sd.off;
    const int ns = P.n_stages;
    for (int gi = 0; gi < ngroups; ++gi) {
      const int gp = min(sh.g, sd.nrows - gi * sh.g);
      const unsigned bytes = (unsigned)gp * sh.kc * 2u;
      const unsigned char* gsrc = base + (size_t)gi * sh.g * sh.K * 2;
      for (int kj = 0; kj < sh.nk; ++kj) {
        const int s = (int)(t % ns);
        const unsigned n = t / ns;
        if (n > 0 && !wait_bar(P, sc, &sc->empty[s], (n - 1) & 1u, 3, step)) return false;
        mbar_expect_tx(&sc->full[s], bytes);
        bulk_g2s(ring + (size_t)s * kStageBytes, gsrc + (size_t)kj * bytes, bytes, &sc->full[s], pol);
        ++t;
      }
    }
    return true;
  }

  __device__ void run() {
    const int c = blockIdx.x;
    const SegDesc* D = P.desc + (size_t)c * (P.L * P.slots + 1);
    bool ok = true;
    unsigned route_round = 0;
    for (step = 0; ok && step < P.n_steps; ++step) {
      for (int l = 0; ok && l < P.L; ++l) {
        const SegDesc* Dl = D + (size_t)l * P.slots;
        ok = issue(Dl[0], P.shp[SK_QKV]) && issue(Dl[1], P.shp[SK_O]);
        if (!ok) break;
        if (P.E == 0) {
          ok = issue(Dl[2], P.shp[SK_GU]) && issue(Dl[3], P.shp[SK_DOWN]);
        } else {
          ok = issue(Dl[2], P.shp[SK_SGU]);
          if (!ok) break;
          // the routed experts are known only once the consumers have run the router
          ok = wait_bar(P, sc, &sc->route_bar, route_round & 1u, 4, step);
          ++route_round;
          if (!ok) break;
          int e[kMaxTopK];
          for (int k = 0; k < P.top_k; ++k) e[k] = sc->route_e[k];
          for (int k = 0; ok && k < P.top_k; ++k) ok = issue(Dl[4 + e[k]], P.shp[SK_EGU]);
          ok = ok && issue(Dl[3], P.shp[SK_SDOWN]);
          for (int k = 0; ok && k < P.top_k; ++k) ok = issue(Dl[4 + P.E + e[k]], P.shp[SK_EDOWN]);
        }
      }
      if (ok && step >= P.lm_from_step) ok = issue(D[(size_t)P.L * P.slots], P.shp[SK_LM]);
    }
    // let every copy still in flight land before the CTA may exit
    const int ns = P.n_stages;
    for (unsigned tt = (t > (unsigned)ns ? t - ns : 0u); tt < t; ++tt) {
      const int s = (int)(tt % ns);
      const unsigned long long t0 = gtimer();
      while (!mbar_test(&sc->full[s], (tt / ns) & 1u)) {
        if (gtimer() - t0 > P.timeout_ns) break;
      }
    }
  }
};

// ---------------------------------------------------------------- consumer

// One tile: G rows x nch 16-byte chunks, row-major in the stage. Lane l takes
// chunks l, l+32, ...; the input vector chunk is read once and reused for all
// G rows. Writes the G row partial sums to part[prow(r)].
template <int G>
__device__ __forceinline__ void tile_gemv(const uint4* __restrict__ w, const float4* __restrict__ xv,
                                          int nch, int lane, float* part, int pidx0, int pstride) {
  float acc[G];
#pragma unroll
  for (int r = 0; r < G; ++r) acc[r] = 0.f;
#pragma unroll 2
  for (int c = lane; c < nch; c += 32) {
    const float4 a = xv[2 * c];
    const float4 b = xv[2 * c + 1];
#pragma unroll
    for (int r = 0; r < G; ++r) acc[r] = dot8(w[r * nch + c], a, b, acc[r]);
  }
  __syncwarp();
#pragma unroll
  for (int r = 0; r < G; ++r) {
    const float v = warp_sum(acc[r]);
    if (lane == r) part[pidx0 + r * pstride] = v;
  }
}

struct Consumer {
  const Params& P;
  SmemCtl* sc;
  float* part;
  float* vec;
  unsigned char* ring;
  const int tid, warp, lane;
  unsigned tbase = 0;   // ring position (tiles consumed by the CTA so far)
  unsigned bar_no = 0;  // grid barriers passed
  int step = 0;
  unsigned route_round = 0;

  __device__ Consumer(const Params& p, SmemCtl* s, float* pa, float* v, unsigned char* r)
      : P(p), sc(s), part(pa), vec(v), ring(r), tid(threadIdx.x), warp(threadIdx.x >> 5),
        lane(threadIdx.x & 31) {}

  __device__ float block_sum(float v) {
    v = warp_sum(v);
    if (lane == 0) sc->red[warp] = v;
    cbar();
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < kConsumerWarps; ++i) t += sc->red[i];
    cbar();
    return t;
  }

  // vec[0..n) = src (fp32, L2-resident scratch)
  __device__ void load_vec(const float* src, int n) {
    for (int i = tid * 4; i < n; i += kConsumerThreads * 4)
      *reinterpret_cast<float4*>(vec + i) = *reinterpret_cast<const float4*>(src + i);
    cbar();
  }

  // vec = RMSNorm(src) * gain, src either fp32 (residual) or an fp16 embedding row.
  __device__ void load_norm(const float* srcf, const __half* srch, const __half* gain, int n) {
    float ss = 0.f;
    if (srcf) {
      for (int i = tid * 4; i < n; i += kConsumerThreads * 4) {
        const float4 v = *reinterpret_cast<const float4*>(srcf + i);
        *reinterpret_cast<float4*>(vec + i) = v;
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
      }
    } else {
      for (int i = tid * 8; i < n; i += kConsumerThreads * 8) {
        const uint4 raw = *reinterpret_cast<const uint4*>(srch + i);
        const __half2* hh = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __half22float2(hh[k]);
          vec[i + 2 * k] = f.x;
          vec[i + 2 * k + 1] = f.y;
          ss = fmaf(f.x, f.x, ss);
          ss = fmaf(f.y, f.y, ss);
        }
      }
    }
    const float tot = block_sum(ss);
    const float inv = 1.0f / sqrtf(tot / (float)n + P.eps);
    for (int i = tid; i < n; i += kConsumerThreads) vec[i] = vec[i] * inv * __half2float(gain[i]);
    cbar();
  }

  // Consume one segment's tiles; partial sums land in part[pbase + row*pstride + kjbase + kj].
  __device__ void run_segment(const SegDesc& sd, const SegShape& sh, const float* vseg, int pbase,
                              int pstride, int kjbase) {
    const int ngroups = (sd.nrows + sh.g - 1) / sh.g;
    const int ntiles = ngroups * sh.nk;
    const int ns = P.n_stages;
    const int nch = sh.kc / 8;
    for (int i = warp; i < ntiles; i += kConsumerWarps) {
      if (sc->abort) break;
      const unsigned t = tbase + i;
      const int s = (int)(t % ns);
      if (!wait_bar(P, sc, &sc->full[s], (t / ns) & 1u, 2, step)) break;
      const int gi = i / sh.nk, kj = i - gi * sh.nk;
      const int gp = min(sh.g, sd.nrows - gi * sh.g);
      const uint4* w = reinterpret_cast<const uint4*>(ring + (size_t)s * kStageBytes);
      const float4* xv = reinterpret_cast<const float4*>(vseg + (size_t)kj * sh.kc);
      const int p0 = pbase + gi * sh.g * pstride + kjbase + kj;
      // the stage is released inside tile_gemv's reduction (after __syncwarp)
      switch (gp) {
        case 1: tile_gemv<1>(w, xv, nch, lane, part, p0, pstride); break;
        case 2: tile_gemv<2>(w, xv, nch, lane, part, p0, pstride); break;
        case 3: tile_gemv<3>(w, xv, nch, lane, part, p0, pstride); break;
        case 4: tile_gemv<4>(w, xv, nch, lane, part, p0, pstride); break;
        case 5: tile_gemv<5>(w, xv, nch, lane, part, p0, pstride); break;
        case 6: tile_gemv<6>(w, xv, nch, lane, part, p0, pstride); break;
        case 7: tile_gemv<7>(w, xv, nch, lane, part, p0, pstride); break;
        default: tile_gemv<8>(w, xv, nch, lane, part, p0, pstride); break;
      }
      if (lane == 0) mbar_arrive(&sc->empty[s]);
    }
    tbase += ntiles;
  }

  __device__ float row_sum(int r, int stride) const {
    float y = 0.f;
    for (int k = 0; k < stride; ++k) y += part[r * stride + k];
    return y;
  }

  // Grid-wide barrier between dependent phases. Returns false if the run aborted.
  __device__ bool grid_sync() {
    cbar();
    if (tid == 0) {
      const unsigned long long ta = P.trace ? gtimer() : 0ull;
      const unsigned k = bar_no++;
      int ab = sc->abort;
      if (ab) {
        atomicExch(&P.ctrl->abort, 1u);
      } else {
        const bool skip = ((int)blockIdx.x == P.fault_cta && (int)k == P.fault_barrier);
        if (!skip) {
          __threadfence();
          red_release_add(&P.ctrl->arrive, 1u);
        }
        const unsigned target = (k + 1) * gridDim.x;
        const unsigned long long t0 = gtimer();
        unsigned it = 0;
        while (ld_acquire(&P.ctrl->arrive) < target) {
          if ((++it & 15) == 0) {
            if (ld_relaxed(&P.ctrl->abort)) {
              ab = 1;
              break;
            }
            if (gtimer() - t0 > P.timeout_ns) {
              record_error(P, kErrTimeout, 1, step);
              ab = 1;
              break;
            }
          }
        }
      }
      if (P.trace && (int)k < P.trace_cap) {
        unsigned long long* tr = P.trace + ((size_t)blockIdx.x * P.trace_cap + k) * 2;
        tr[0] = ta;
        tr[1] = gtimer();
      }
      sc->abort = ab;
    }
    cbar();
    return !sc->abort;
  }

  // ---- attention: split-K over positions, units (kv head, chunk), one warp each
  template <int DH>
  __device__ void attention(int l, int pos) {
    constexpr int DPL = DH / 32;  // dims per lane in the V accumulation
    const int T = pos + 1;
    const int hk = P.hk, hq = P.hq;
    const int nwarps = gridDim.x * kConsumerWarps;
    int pc = (T * hk + nwarps - 1) / nwarps;
    pc = ((max(pc, kAttnSub) + kAttnSub - 1) / kAttnSub) * kAttnSub;
    const int nch = (T + pc - 1) / pc;
    const int units = hk * nch;
    float* qs = vec + warp * (kMaxHeadsPerGroup * DH);
    const float2* rp = P.rope + (size_t)pos * (DH / 2);
    const float scale = rsqrtf((float)DH);
    for (int u = blockIdx.x * kConsumerWarps + warp; u < units; u += nwarps) {
      const int g = u / nch, ch = u - (u / nch) * nch;
      const int h_lo = (g * hq + hk - 1) / hk;
      const int nh = (((g + 1) * hq + hk - 1) / hk) - h_lo;
      // rotated, pre-scaled queries of the group's heads
      for (int hh = 0; hh < nh; ++hh) {
        const float* qr = P.qkv + (size_t)(h_lo + hh) * DH;
        for (int i = lane; i < DH / 2; i += 32) {
          const float a = qr[i], b = qr[i + DH / 2];
          const float2 cs = rp[i];
          qs[hh * DH + i] = (a * cs.x - b * cs.y) * scale;
          qs[hh * DH + i + DH / 2] = (a * cs.y + b * cs.x) * scale;
        }
      }
      __half* Kc = P.kcache + ((size_t)(l * hk + g) * P.max_ctx) * DH;
      __half* Vc = P.vcache + ((size_t)(l * hk + g) * P.max_ctx) * DH;
      if (ch == nch - 1) {  // append this token's rotated k and its v at position pos
        const float* kr = P.qkv + (size_t)hq * DH + (size_t)g * DH;
        const float* vr = P.qkv + (size_t)(hq + hk) * DH + (size_t)g * DH;
        for (int i = lane; i < DH / 2; i += 32) {
          const float a = kr[i], b = kr[i + DH / 2];
          const float2 cs = rp[i];
          Kc[(size_t)pos * DH + i] = __float2half_rn(a * cs.x - b * cs.y);
          Kc[(size_t)pos * DH + i + DH / 2] = __float2half_rn(a * cs.y + b * cs.x);
          Vc[(size_t)pos * DH + i] = __float2half_rn(vr[i]);
          Vc[(size_t)pos * DH + i + DH / 2] = __float2half_rn(vr[i + DH / 2]);
        }
      }
      __syncwarp();
      const int j0 = ch * pc, j1 = min(T, j0 + pc);
      float m[kMaxHeadsPerGroup], ls[kMaxHeadsPerGroup], acc[kMaxHeadsPerGroup][DPL];
#pragma unroll
      for (int hh = 0; hh < kMaxHeadsPerGroup; ++hh) {
        m[hh] = -INFINITY;
        ls[hh] = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[hh][e] = 0.f;
      }
      for (int jb = j0; jb < j1; jb += kAttnSub) {
        const int j = jb + lane;
        const bool valid = j < j1;
        float s[kMaxHeadsPerGroup];
#pragma unroll
        for (int hh = 0; hh < kMaxHeadsPerGroup; ++hh) s[hh] = 0.f;
        if (valid) {
          const uint4* kr = reinterpret_cast<const uint4*>(Kc + (size_t)j * DH);
          uint4 kv[DH / 8];
#pragma unroll
          for (int i = 0; i < DH / 8; ++i) kv[i] = kr[i];
#pragma unroll
          for (int hh = 0; hh < kMaxHeadsPerGroup; ++hh) {
            if (hh < nh) {
              const float4* q4 = reinterpret_cast<const float4*>(qs + hh * DH);
              float a = 0.f;
#pragma unroll
              for (int i = 0; i < DH / 8; ++i) a = dot8(kv[i], q4[2 * i], q4[2 * i + 1], a);
              s[hh] = a;
            }
          }
        }
        float p[kMaxHeadsPerGroup];
#pragma unroll
        for (int hh = 0; hh < kMaxHeadsPerGroup; ++hh) {
          if (hh < nh) {
            const float sv = valid ? s[hh] : -INFINITY;
            const float mn = fmaxf(m[hh], warp_max(sv));
            p[hh] = valid ? expf(sv - mn) : 0.f;
            const float corr = expf(m[hh] - mn);
            ls[hh] = ls[hh] * corr + warp_sum(p[hh]);
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[hh][e] *= corr;
            m[hh] = mn;
          }
        }
        const int nj = min(kAttnSub, j1 - jb);
#pragma unroll 4
        for (int jj = 0; jj < nj; ++jj) {
          const __half* vrow = Vc + (size_t)(jb + jj) * DH + lane * DPL;
          float vv[DPL];
          if constexpr (DPL == 4) {
            const uint2 raw = *reinterpret_cast<const uint2*>(vrow);
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
            const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
            vv[0] = a.x; vv[1] = a.y; vv[2] = b.x; vv[3] = b.y;
          } else {
#pragma unroll
            for (int e = 0; e < DPL; ++e) vv[e] = __half2float(vrow[e]);
          }
#pragma unroll
          for (int hh = 0; hh < kMaxHeadsPerGroup; ++hh) {
            if (hh < nh) {
              const float pj = __shfl_sync(0xffffffffu, p[hh], jj);
#pragma unroll
              for (int e = 0; e < DPL; ++e) acc[hh][e] = fmaf(pj, vv[e], acc[hh][e]);
            }
          }
        }
      }
      // partials (m, l, acc) of this chunk
      const int stride = DH + 4;
#pragma unroll
      for (int hh = 0; hh < kMaxHeadsPerGroup; ++hh) {
        if (hh < nh) {
          float* pb = P.apart + ((size_t)(h_lo + hh) * P.max_chunks + ch) * stride;
          if (lane == 0) {
            pb[0] = m[hh];
            pb[1] = ls[hh];
          }
#pragma unroll
          for (int e = 0; e < DPL; ++e) pb[4 + lane * DPL + e] = acc[hh][e];
        }
      }
      __threadfence();
      __syncwarp();
      unsigned old = 0;
      if (lane == 0) old = atomicAdd(&P.acnt[g], 1u);
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old == (unsigned)(nch - 1)) {  // last chunk of this KV head: combine
        __threadfence();
        for (int hh = 0; hh < nh; ++hh) {
          const float* hb = P.apart + (size_t)(h_lo + hh) * P.max_chunks * stride;
          float M = -INFINITY;
          for (int cc = lane; cc < nch; cc += 32) M = fmaxf(M, __ldcg(hb + (size_t)cc * stride));
          M = warp_max(M);
          float Ls = 0.f, a[DPL];
#pragma unroll
          for (int e = 0; e < DPL; ++e) a[e] = 0.f;
          for (int cc = 0; cc < nch; ++cc) {
            const float* cb = hb + (size_t)cc * stride;
            const float w = expf(__ldcg(cb) - M);
            Ls = fmaf(w, __ldcg(cb + 1), Ls);
#pragma unroll
            for (int e = 0; e < DPL; ++e) a[e] = fmaf(w, __ldcg(cb + 4 + lane * DPL + e), a[e]);
          }
          const float inv = 1.0f / Ls;
#pragma unroll
          for (int e = 0; e < DPL; ++e) P.o[(size_t)(h_lo + hh) * DH + lane * DPL + e] = a[e] * inv;
        }
        if (lane == 0) P.acnt[g] = 0u;
      }
    }
  }

  __device__ void attention_dispatch(int l, int pos) {
    if (P.dh == 128) attention<128>(l, pos);
    else attention<64>(l, pos);
  }

  // residual epilogue: x[row] = xprev[row] + sum of partials
  __device__ void epi_residual(const SegDesc& sd, int stride, const __half* xprev_h) {
    for (int r = tid; r < sd.nrows; r += kConsumerThreads) {
      const int row = sd.row0 + r;
      const float xp = xprev_h ? __half2float(xprev_h[row]) : P.x[row];
      P.x[row] = xp + row_sum(r, stride);
    }
  }

  // SwiGLU epilogue over interleaved (gate, up) rows: h[hoff + row0/2 + j] = w * silu(g) * u
  __device__ void epi_swiglu(const SegDesc& sd, int pbase, int stride, int hoff, float w) {
    const int npairs = sd.nrows / 2;
    for (int j = tid; j < npairs; j += kConsumerThreads) {
      float yg = 0.f, yu = 0.f;
      for (int k = 0; k < stride; ++k) {
        yg += part[pbase + (2 * j) * stride + k];
        yu += part[pbase + (2 * j + 1) * stride + k];
      }
      P.h[hoff + sd.row0 / 2 + j] = w * silu(yg) * yu;
    }
  }

  // MoE router, computed redundantly by every CTA from the normalised input in vec.
  __device__ void route(int l) {
    const __half* R = P.router + (size_t)l * P.E * P.d;
    for (int e = warp; e < P.E; e += kConsumerWarps) {
      const __half* row = R + (size_t)e * P.d;
      float a = 0.f;
      for (int c = lane; c < P.d / 8; c += 32) {
        const uint4 wv = *reinterpret_cast<const uint4*>(row + c * 8);
        a = dot8(wv, *reinterpret_cast<const float4*>(vec + c * 8),
                 *reinterpret_cast<const float4*>(vec + c * 8 + 4), a);
      }
      a = warp_sum(a);
      if (lane == 0) part[e] = a;
    }
    cbar();
    if (tid == 0) {
      float mx = -INFINITY;
      for (int e = 0; e < P.E; ++e) mx = fmaxf(mx, part[e]);
      float* pr = part + kMaxExperts;  // softmax numerators (the denominator cancels below)
      for (int e = 0; e < P.E; ++e) pr[e] = expf(part[e] - mx);
      unsigned long long used = 0ull;
      float wsum = 0.f;
      for (int k = 0; k < P.top_k; ++k) {
        int bi = -1;
        float bv = -INFINITY;
        for (int e = 0; e < P.E; ++e)
          if (!((used >> e) & 1ull) && (bi < 0 || pr[e] > bv)) {
            bi = e;
            bv = pr[e];
          }
        used |= 1ull << bi;
        sc->route_e[k] = bi;
        sc->route_w[k] = bv;
        wsum += bv;
      }
      for (int k = 0; k < P.top_k; ++k) sc->route_w[k] /= wsum;
      mbar_arrive(&sc->route_bar);  // hand the choice to the producer
    }
    cbar();
  }

  __device__ bool layer(int l, int tok, int pos, const SegDesc* D) {
    const SegDesc* Dl = D + (size_t)l * P.slots;
    const __half* erow = P.embed + (size_t)tok * P.d;
    // ---- q, k, v projections of RMSNorm(x)
    if (l == 0) load_norm(nullptr, erow, P.attn_norm, P.d);
    else load_norm(P.x, nullptr, P.attn_norm + (size_t)l * P.d, P.d);
    const SegShape& sq = P.shp[SK_QKV];
    run_segment(Dl[0], sq, vec, 0, sq.nk, 0);
    cbar();
    for (int r = tid; r < Dl[0].nrows; r += kConsumerThreads) P.qkv[Dl[0].row0 + r] = row_sum(r, sq.nk);
    if (!grid_sync()) return false;
    // ---- RoPE, KV append, attention
    attention_dispatch(l, pos);
    if (!grid_sync()) return false;
    // ---- output projection + residual
    load_vec(P.o, P.hq * P.dh);
    const SegShape& so = P.shp[SK_O];
    run_segment(Dl[1], so, vec, 0, so.nk, 0);
    cbar();
    epi_residual(Dl[1], so.nk, l == 0 ? erow : nullptr);
    if (!grid_sync()) return false;
    // ---- FFN
    load_norm(P.x, nullptr, P.mlp_norm + (size_t)l * P.d, P.d);
    if (P.E == 0) {
      const SegShape& sg = P.shp[SK_GU];
      run_segment(Dl[2], sg, vec, 0, sg.nk, 0);
      cbar();
      epi_swiglu(Dl[2], 0, sg.nk, 0, 1.0f);
      if (!grid_sync()) return false;
      load_vec(P.h, P.ff);
      const SegShape& sd = P.shp[SK_DOWN];
      run_segment(Dl[3], sd, vec, 0, sd.nk, 0);
      cbar();
      epi_residual(Dl[3], sd.nk, nullptr);
      if (!grid_sync()) return false;
    } else {
      route(l);
      int e[kMaxTopK];
      float w[kMaxTopK];
      for (int k = 0; k < P.top_k; ++k) {
        e[k] = sc->route_e[k];
        w[k] = sc->route_w[k];
      }
      const SegShape& ss = P.shp[SK_SGU];
      const SegShape& se = P.shp[SK_EGU];
      const SegDesc& dsh = Dl[2];
      run_segment(dsh, ss, vec, 0, ss.nk, 0);
      int pb[kMaxTopK];
      int pnext = dsh.nrows * ss.nk;
      for (int k = 0; k < P.top_k; ++k) {
        pb[k] = pnext;
        const SegDesc& de = Dl[4 + e[k]];
        run_segment(de, se, vec, pb[k], se.nk, 0);
        pnext += de.nrows * se.nk;
      }
      cbar();
      epi_swiglu(dsh, 0, ss.nk, 0, 1.0f);
      for (int k = 0; k < P.top_k; ++k) epi_swiglu(Dl[4 + e[k]], pb[k], se.nk, P.ffs + k * P.ffe, w[k]);
      if (!grid_sync()) return false;
      load_vec(P.h, P.ffs + P.top_k * P.ffe);
      const SegShape& sds = P.shp[SK_SDOWN];
      const SegShape& sde = P.shp[SK_EDOWN];
      const int stride = sds.nk + P.top_k * sde.nk;
      run_segment(Dl[3], sds, vec, 0, stride, 0);
      for (int k = 0; k < P.top_k; ++k)
        run_segment(Dl[4 + P.E + e[k]], sde, vec + P.ffs + k * P.ffe, 0, stride, sds.nk + k * sde.nk);
      cbar();
      epi_residual(Dl[3], stride, nullptr);
      if (!grid_sync()) return false;
    }
    return true;
  }

  __device__ void run() {
    const int c = blockIdx.x;
    const SegDesc* D = P.desc + (size_t)c * (P.L * P.slots + 1);
    int tok = P.first_token;
    for (step = 0; step < P.n_steps; ++step) {
      const int pos = P.pos0 + step;
      if (tok < 0 || tok >= P.V) {
        if (tid == 0) record_error(P, kErrDevice, 5, step);
        return;
      }
      for (int l = 0; l < P.L; ++l)
        if (!layer(l, tok, pos, D)) return;
      int next;
      if (step >= P.lm_from_step) {
        // ---- final norm, LM head, greedy argmax
        load_norm(P.x, nullptr, P.final_norm, P.d);
        const SegDesc& dl = D[(size_t)P.L * P.slots];
        const SegShape& sl = P.shp[SK_LM];
        run_segment(dl, sl, vec, 0, sl.nk, 0);
        cbar();
        float v1 = -INFINITY, v2 = -INFINITY;
        int i1 = INT_MAX;
        for (int r = tid; r < dl.nrows; r += kConsumerThreads) {
          const float y = row_sum(r, sl.nk);
          const int row = dl.row0 + r;
          if (P.logits_out) P.logits_out[(size_t)step * P.V + row] = y;
          cand_merge(v1, i1, v2, y, row, -INFINITY);
        }
        cand_warp_merge(v1, i1, v2);
        if (lane == 0) sc->wcand[warp] = Cand{v1, i1, v2, 0};
        cbar();
        if (tid == 0) {
          float a1 = -INFINITY, a2 = -INFINITY;
          int ai = INT_MAX;
          for (int w = 0; w < kConsumerWarps; ++w)
            cand_merge(a1, ai, a2, sc->wcand[w].v1, sc->wcand[w].i1, sc->wcand[w].v2);
          P.cand[c] = Cand{a1, ai, a2, 0};
        }
        if (!grid_sync()) return;
        v1 = -INFINITY;
        v2 = -INFINITY;
        i1 = INT_MAX;
        for (int cc = tid; cc < (int)gridDim.x; cc += kConsumerThreads) {
          const float b1 = __ldcg(&P.cand[cc].v1);
          const int bi = __ldcg(&P.cand[cc].i1);
          const float b2 = __ldcg(&P.cand[cc].v2);
          cand_merge(v1, i1, v2, b1, bi, b2);
        }
        cand_warp_merge(v1, i1, v2);
        if (lane == 0) sc->wcand[warp] = Cand{v1, i1, v2, 0};
        cbar();
        if (tid == 0) {
          float a1 = -INFINITY, a2 = -INFINITY;
          int ai = INT_MAX;
          for (int w = 0; w < kConsumerWarps; ++w)
            cand_merge(a1, ai, a2, sc->wcand[w].v1, sc->wcand[w].i1, sc->wcand[w].v2);
          sc->tok = ai;
          sc->margin = a1 - a2;
          if (c == 0) {
            P.out_tokens[step] = ai;
            if (P.margins_out) P.margins_out[step] = a1 - a2;
          }
        }
        cbar();
        next = sc->tok;
        if (next == INT_MAX) {  // no finite logit
          if (tid == 0) record_error(P, kErrDevice, 5, step);
          return;
        }
        if (P.forced && P.forced[step] >= 0) next = P.forced[step];
      } else {
        next = P.forced ? P.forced[step] : -1;
      }
      tok = next;
    }
    if (c == 0 && tid == 0) P.ctrl->final_token = tok;
  }
};

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) unsigned char smem[];
  SmemCtl* sc = reinterpret_cast<SmemCtl*>(smem);
  float* part = reinterpret_cast<float*>(smem + smem_ctl_bytes());
  float* vec = part + kPartFloats;
  unsigned char* ring = smem + smem_ring_offset(P.vec_floats);
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.n_stages; ++s) {
      mbar_init(&sc->full[s], 1);
      mbar_init(&sc->empty[s], 1);
    }
    mbar_init(&sc->route_bar, 1);
    sc->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x >= kConsumerThreads) {
    if (threadIdx.x == kConsumerThreads) {
      Producer pr(P, sc, ring);
      pr.run();
    }
    return;
  }
  Consumer cs(P, sc, part, vec, ring);
  cs.run();
}

// ---- host-side accessors used by the launcher
int kernel_smem_bytes(int vec_floats, int n_stages) { return smem_total(vec_floats, n_stages); }
int kernel_max_stages() { return kMaxStages; }
const void* kernel_entry() { return reinterpret_cast<const void*>(&decode_kernel); }

}  // namespace kie
