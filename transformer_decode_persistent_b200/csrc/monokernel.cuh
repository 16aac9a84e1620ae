// Persistent batch-1 decode kernel for B200 (sm_100a).
//
// One cooperative launch runs n whole decode steps: every matrix product, the
// attention, the normalisations and the token choice stay inside one
// GPU-resident program that feeds each new token back to itself without a
// return to the host ("メモリの壁を打破する：標準的なGPUで3,000 tokens/sの推論を
// 実現する", section "1. The Monokernel Runtime"). At batch 1 a step is bound by
// moving every active weight from HBM once per token (same page, section
// "ボトルネック：計算量ではなくメモリ帯域幅"), so the kernel is organised around
// keeping HBM busy and the dependency chain short:
//
//  * One CTA per SM. Each CTA owns a contiguous region of a packed "weight
//    tape" that holds, in execution order, its slice of every matrix of one
//    decode step (see kie_internal.h for the tile format).
//  * Warp 7 of each CTA is the producer: lanes 0..13 each own one of 14
//    shared-memory ring stages and stream the CTA's tape tiles (and attention
//    K/V rows) into it with TMA bulk copies (cp.async.bulk, L2 evict-first),
//    completion tracked by mbarriers. It never waits on the consumers' data
//    dependencies, so the next phase's weights are in flight while the current
//    phase finishes.
//  * Warps 0-6 are consumers: GEMV on each tile against the fp32 input vector
//    held in shared memory (fp16 weights, fp32 FMA), RMSNorm (recomputed by
//    every CTA), RoPE, split-K attention over the fp16 KV cache, SwiGLU,
//    residual adds, the LM head and a greedy argmax.
//  * Phases exchange data through flagged 64-bit words (value and the epoch of
//    the phase that wrote it): a phase waits only for the words it reads, so
//    there is no grid-wide barrier between phases. One grid barrier per step
//    orders the step's KV-cache appends before the next step's bulk copies.
//    This is where the per-operation synchronisation cost that the pages
//    name (same page, section "マイクロ秒が失われる場所") is removed.
//
// Every wait (flagged words, step barrier, ring stages, routing hand-off) is
// bounded: on a deadline the kernel records KIE_ERR_TIMEOUT in the control
// block, raises an abort flag that all CTAs poll, lets in-flight bulk copies
// land, and returns.
#include <cuda_fp16.h>
#include <float.h>
#include <limits.h>
#include <stdint.h>

#include "kie_internal.h"

namespace kie {

constexpr int kMaxStages = kRingStages;
constexpr int kErrTimeout = -5;  // KIE_ERR_TIMEOUT
constexpr int kErrDevice = -6;   // KIE_ERR_DEVICE

constexpr int kRouteRing = 8;  // routing decisions kept for lagging issuer lanes
constexpr int kRopeStage = 128; // RoPE pairs whose coefficients are staged in shared memory

struct SmemCtl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  volatile int abort;
  volatile unsigned route_seq;  // routing decisions published so far
  int tok;
  float margin;
  int route_e[kRouteRing][kMaxTopK];
  float route_w[kMaxTopK];
  float red[64];
  float ssq[kConsumerWarps];  // per-warp sums of squares of the last RMSNorm input
  float2 rcs[kRopeStage];     // RoPE (cos, sin) of this CTA's first q/k pairs at this step's position
  unsigned sel_hist[256];     // sampling: radix-select histogram
  unsigned long long sel_key[kSampleK];  // sampling: the selected top-k keys, then sorted
  unsigned long long sel_prefix;
  int sel_need, sel_count;
  Cand wcand[kConsumerWarps];
  unsigned bcast;
  // this CTA's rows of the residual stream: the output projection and the
  // FFN down projection own the same rows in every layer
  float xown[kMaxOwnRows];
};

// Shared-memory layout, identical on host and device.
__host__ __device__ inline int smem_ctl_bytes() { return (int)((sizeof(SmemCtl) + 127) & ~127); }
// control block | partial sums | vector buffer | descriptor cache | ring
__host__ __device__ inline int smem_desc_offset(int vec_floats) {
  return (smem_ctl_bytes() + kPartFloats * 4 + vec_floats * 4 + 15) & ~15;
}
__host__ __device__ inline int smem_ring_offset(int vec_floats, int n_desc) {
  const int b = smem_desc_offset(vec_floats) + n_desc * (int)sizeof(SegDesc);
  return (b + 1023) & ~1023;
}
__host__ __device__ inline int smem_total(int vec_floats, int n_desc, int n_stages, int stage_bytes) {
  return smem_ring_offset(vec_floats, n_desc) + n_stages * stage_bytes;
}

// This CTA's descriptors of the per-layer segments q/k/v, o, gate/up and down
// (slots 0..3) and of the LM head, copied to shared memory at launch so that a
// phase does not start with a global load. Routed experts' descriptors stay in
// global memory.
struct DescCache {
  const SegDesc* sm;  // [4 L + 1]
  const SegDesc* g;   // this CTA's global descriptors [L * slots + 1]
  int L, slots;
  __device__ __forceinline__ const SegDesc& at(int l, int slot) const {
    if (l == L) return sm[4 * L];
    return slot < 4 ? sm[4 * l + slot] : g[(size_t)l * slots + slot];
  }
};

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
// non-blocking probe of an mbarrier phase (never suspends the thread)
__device__ __forceinline__ bool mbar_probe(uint64_t* b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
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
// ---- flagged words: float value in the low half, writer's epoch in the high half
__device__ __forceinline__ unsigned long long fpack(float v, unsigned ep) {
  return ((unsigned long long)ep << 32) | __float_as_uint(v);
}
__device__ __forceinline__ void st_flag(unsigned long long* p, float v, unsigned ep) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(fpack(v, ep)) : "memory");
}
__device__ __forceinline__ void st_flag2(unsigned long long* p, float a, float b, unsigned ep) {
  asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(fpack(a, ep)), "l"(fpack(b, ep))
               : "memory");
}
__device__ __forceinline__ void ld_flag2(const unsigned long long* p, unsigned long long& a,
                                         unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
__device__ __forceinline__ unsigned long long ld_flag1(const unsigned long long* p) {
  unsigned long long a;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(a) : "l"(p) : "memory");
  return a;
}
__device__ __forceinline__ unsigned fepoch(unsigned long long w) { return (unsigned)(w >> 32); }
__device__ __forceinline__ float fval(unsigned long long w) { return __uint_as_float((unsigned)w); }
// consumer-only barrier (named barrier 1 over the 224 consumer threads)
__device__ __forceinline__ void cbar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}
// consumer barrier that also ORs a predicate over the consumer threads, so
// that all of them take the same branch on it
__device__ __forceinline__ bool cbar_any(bool v) {
  unsigned r;
  asm volatile(
      "{\n.reg .pred p, q;\nsetp.ne.u32 p, %1, 0;\nbar.red.or.pred q, 1, %2, p;\nselp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((unsigned)v), "n"(kConsumerThreads)
      : "memory");
  return r != 0;
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
// two packed fp16 values (by value, so register arrays stay in registers)
__device__ __forceinline__ float2 h2f2(unsigned u) {
  __half2 h;
  memcpy(&h, &u, sizeof(h));
  return __half22float2(h);
}
// two floats (already fp16-exact) as the bits of a half2
__device__ __forceinline__ uint32_t f2h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}

// Explicit shared-memory loads by 32-bit shared address: the ring and the
// input vector are reached through pointers kept in the consumer's state, and
// generic loads of shared memory are slower than ld.shared.
__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ float4 lds_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}

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

// Butterfly transpose-reduction: lane l holds v[j] = its share of the dot
// product of position j; afterwards v[0] of lane l is the full sum for j = l.
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const bool up = lane & 16;
    const float send = up ? v[k] : v[k + 16];
    const float keep = up ? v[k + 16] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const bool up = lane & 8;
    const float send = up ? v[k] : v[k + 8];
    const float keep = up ? v[k + 8] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const bool up = lane & 4;
    const float send = up ? v[k] : v[k + 4];
    const float keep = up ? v[k + 4] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool up = lane & 2;
    const float send = up ? v[k] : v[k + 2];
    const float keep = up ? v[k + 2] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  {
    const bool up = lane & 1;
    const float send = up ? v[0] : v[1];
    const float keep = up ? v[1] : v[0];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
  return v[0];
}

// N values per lane (N a power of two up to 16) summed over the warp: lane l
// ends with the warp total of value (l mod N). Butterfly on the low lane bits,
// then plain sums over the remaining bits.
template <int N>
__device__ __forceinline__ float transpose_reduce(float (&v)[N], int lane) {
#pragma unroll
  for (int o = N / 2; o >= 1; o /= 2) {
    const bool up = lane & o;
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float send = up ? v[k] : v[k + o];
      const float keep = up ? v[k + o] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = N; o < 32; o *= 2) r += __shfl_xor_sync(0xffffffffu, r, o);
  return r;
}

// ---------------------------------------------------------------- sampling helpers

// Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC 2011): ten rounds of two 32x32->64-bit products on the
// counter words, the key bumped by the Weyl constants between rounds. Returns
// the first output word.
__device__ __forceinline__ uint32_t philox_w0(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                              uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

// Sampling order key: larger logit first, then lower index. The float maps to
// an unsigned integer with the same order; the index is stored inverted.
__device__ __forceinline__ unsigned long long sample_key(float v, int idx) {
  const unsigned b = __float_as_uint(v);
  const unsigned o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((unsigned long long)o << 32) | (0xFFFFFFFFu - (unsigned)idx);
}
__device__ __forceinline__ float key_value(unsigned long long k) {
  const unsigned o = (unsigned)(k >> 32);
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}
__device__ __forceinline__ int key_index(unsigned long long k) { return (int)(0xFFFFFFFFu - (unsigned)k); }

// ---------------------------------------------------------------- errors

static __device__ void record_error(const Params& P, int code, int where, int step) {
  if (atomicCAS(&P.ctrl->err, 0, code) == 0) {
    P.ctrl->err_cta = blockIdx.x;
    P.ctrl->err_step = step;
    P.ctrl->err_where = where;
  }
  __threadfence();
  atomicExch(&P.ctrl->abort, 1u);
}

// Bounded wait on an mbarrier phase. Returns false on abort or deadline.
// `spin` waits with non-suspending probes: the producer's issuer lanes share
// one warp and wait on different stages, and a lane suspended in try_wait
// would hold up the others.
static __device__ bool wait_bar(const Params& P, SmemCtl* sc, uint64_t* b, unsigned parity, int where,
                         int step, bool spin = false) {
  if (spin ? mbar_probe(b, parity) : mbar_test(b, parity)) return true;
  const unsigned long long t0 = gtimer();
  for (unsigned it = 1;; ++it) {
    if (spin ? mbar_probe(b, parity) : mbar_test(b, parity)) return true;
    if ((it & 63) == 0) {
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

// ---------------------------------------------------------------- attention plan
// Attention work for one layer at position pos (T = pos + 1 keys): units are
// (KV head g, chunk of `per` positions), unit u handled by CTA u % grid. The
// chunk length is about T hk / grid rounded up to whole warp sub-ranges, and
// is lengthened when that would leave a few units over for a second wave; each
// of the kConsumerWarps warps of a unit takes pw = per / kConsumerWarps
// positions as nsb sub-blocks of 32. The K and V rows of every sub-block are
// streamed through the ring like weight tiles: per (unit, sub-block round) the
// ring carries 7 K tiles (sub-ranges 0..6) and then 7 V tiles, so that both
// tiles of sub-range k land on the same consumer warp. The row of `pos` itself
// is written during this step and is never in a tile; the warp that owns it
// reads it directly.
//
// A unit is normally one KV head's chunk for all the query heads it serves
// (its K/V rows are read once); a group of more than kMaxHeadsPerGroup query
// heads is cut into `sub` equal sub-units of at most that many (each reads the
// group's K/V rows). When the query heads' units of every chunk fit in one
// wave of CTAs (short context with grouped heads), each query head becomes a
// unit of its own instead: the group's K/V rows are then read once per query
// head, a small cost at short context, and the work of a group is spread over
// as many CTAs as it has query heads. Per head the arithmetic and its order
// are the same either way.
struct AttnPlan {
  int T, per, pw, nsb, nchk, units, split, sub, hs;
};
__device__ __forceinline__ AttnPlan attn_plan(int pos, int hk, int hq, int grid) {
  constexpr int kUnitMin = kConsumerWarps * kAttnSub;
  AttnPlan a;
  a.T = pos + 1;
  int per = (int)(((long long)a.T * hk + grid - 1) / grid);
  per = ((max(per, kUnitMin) + kUnitMin - 1) / kUnitMin) * kUnitMin;
  const int gmax = (hq + hk - 1) / hk;  // query heads of the largest group
  a.sub = (gmax + kMaxHeadsPerGroup - 1) / kMaxHeadsPerGroup;
  a.hs = (gmax + a.sub - 1) / a.sub;
  // a unit count just past the grid would leave a few CTAs with two units and
  // every layer waiting for them: then take the most chunks that fit one wave
  // (longer units, none doubled)
  const int upc = hk * a.sub;  // units per chunk
  if (upc * ((a.T + per - 1) / per) > grid && grid >= upc) {
    const int nmax = grid / upc;
    per = (a.T + nmax - 1) / nmax;
    per = ((per + kUnitMin - 1) / kUnitMin) * kUnitMin;
  }
  a.per = per;
  a.pw = per / kConsumerWarps;
  a.nsb = a.pw / kAttnSub;
  a.nchk = (a.T + per - 1) / per;
  a.split = (hq > hk && hq * a.nchk <= grid) ? 1 : 0;
  a.units = (a.split ? hq : upc) * a.nchk;
  return a;
}
// Unit u: KV head g, chunk ch, query heads h_lo .. h_lo + nh - 1. KV head g
// serves query heads ceil(g hq / hk) .. ceil((g + 1) hq / hk) - 1, so query
// head q belongs to KV head floor(q hk / hq). The host admits only shapes in
// which every sub-unit gets at least one query head.
struct AttnUnit {
  int g, ch, h_lo, nh;
};
__device__ __forceinline__ AttnUnit attn_unit(const AttnPlan& a, int u, int hk, int hq) {
  AttnUnit r;
  const int idx = u / a.nchk;
  r.ch = u - idx * a.nchk;
  if (a.split) {
    r.h_lo = idx;
    r.nh = 1;
    r.g = (int)(((long long)idx * hk) / hq);
  } else {
    r.g = idx / a.sub;
    const int sgi = idx - r.g * a.sub;
    const int glo = (r.g * hq + hk - 1) / hk, ghi = ((r.g + 1) * hq + hk - 1) / hk;
    r.h_lo = glo + sgi * a.hs;
    r.nh = min(ghi, r.h_lo + a.hs) - r.h_lo;
  }
  return r;
}
__device__ __forceinline__ int attn_units_of(const AttnPlan& a, int cta, int grid) {
  return a.units > cta ? (a.units - cta + grid - 1) / grid : 0;
}
constexpr int kAttnTilesPerRound = 2 * kConsumerWarps;

// ---------------------------------------------------------------- producer

template <bool MOE>
struct Producer {
  // Each of the producer warp's lanes 0..n_stages-1 owns one ring stage and
  // issues the bulk copies of the tiles that land in it (tile t -> stage
  // t % n_stages). A bulk copy occupies its issuing thread for roughly one
  // memory round trip, so one issuer per stage keeps n_stages copies in flight.
  const Params& P;
  SmemCtl* sc;
  unsigned char* ring;
  unsigned long long pol;
  const int lane;
  unsigned t = 0;     // tiles walked (all lanes walk the same sequence)
  unsigned mine = 0;  // tiles issued by this lane
  int step = 0;

  const DescCache dc;

  __device__ Producer(const Params& p, SmemCtl* s, unsigned char* r, int ln, const DescCache& d)
      : P(p), sc(s), ring(r), lane(ln), dc(d) {
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  }

  // Put tile tt (bytes at src; 0 bytes = an empty tile) into this lane's stage.
  __device__ bool put(unsigned tt, const void* src, unsigned bytes) {
    const unsigned n = tt / P.n_stages;
    if (n > 0 && !wait_bar(P, sc, &sc->empty[lane], (n - 1) & 1u, 3, step)) return false;
    mbar_expect_tx(&sc->full[lane], bytes);  // with 0 bytes this arrival completes the phase
    if (bytes) bulk_g2s(ring + (size_t)lane * P.stage_bytes, src, bytes, &sc->full[lane], pol);
    ++mine;
    return true;
  }

  __device__ bool issue(const SegDesc& sd, const SegShape& sh) {
    const int ngroups = (sd.nrows + sh.g - 1) / sh.g;
    const int ntiles = ngroups * sh.nk;
    const int ns = P.n_stages;
    const unsigned char* base = P.tape + sd.off;
    // first tile of this segment that lands in this lane's stage
    for (int i = (int)((lane + ns - (int)(t % ns)) % ns); i < ntiles; i += ns) {
      const int gi = i / sh.nk, kj = i - gi * sh.nk;
      const int gp = min(sh.g, sd.nrows - gi * sh.g);
      const unsigned bytes = (unsigned)gp * sh.kc * 2u;
      const unsigned char* src = base + (size_t)gi * sh.g * sh.K * 2 + (size_t)kj * bytes;
      if (!put(t + i, src, bytes)) return false;
    }
    t += ntiles;
    return true;
  }

  // K/V rows of this CTA's attention units of layer l (see attn_plan).
  __device__ bool issue_attn(int l, int pos) {
    const int G = gridDim.x, ns = P.n_stages, hk = P.hk, dh = P.dh;
    const AttnPlan ap = attn_plan(pos, hk, P.hq, G);
    const int nu = attn_units_of(ap, blockIdx.x, G);
    const int per_unit = ap.nsb * kAttnTilesPerRound;
    const int ntiles = nu * per_unit;
    // The cache rows were written with generic stores by other CTAs in earlier
    // steps (ordered before this point by the step barrier and the ring's
    // mbarriers); order them before this lane's bulk (async-proxy) reads.
    if (ntiles > 0) asm volatile("fence.proxy.async.global;" ::: "memory");
    for (int i = (int)((lane + ns - (int)(t % ns)) % ns); i < ntiles; i += ns) {
      const int uo = i / per_unit, r = i - uo * per_unit;
      const int b = r / kAttnTilesPerRound, ti = r - b * kAttnTilesPerRound;
      const int k = ti % kConsumerWarps;
      const bool isv = ti >= kConsumerWarps;
      const int u = blockIdx.x + uo * G;
      const AttnUnit au = attn_unit(ap, u, hk, P.hq);
      const int g = au.g, ch = au.ch;
      const int j0 = ch * ap.per, j1 = min(ap.T, j0 + ap.per);
      const int wj0 = j0 + k * ap.pw, wj1 = min(j1, wj0 + ap.pw);
      const int jb = wj0 + b * kAttnSub;
      const int rows = max(0, min(min(jb + kAttnSub, wj1), pos) - jb);
      const __half* cache = (isv ? P.vcache : P.kcache) + ((size_t)(l * hk + g) * P.max_ctx + jb) * dh;
      if (!put(t + i, cache, (unsigned)rows * dh * 2u)) return false;
    }
    t += ntiles;
    return true;
  }

  // Spin until the consumers have published routing decision `round`.
  __device__ bool wait_route(unsigned round) {
    const unsigned long long t0 = gtimer();
    for (unsigned it = 0; sc->route_seq <= round; ++it) {
      if ((it & 63) == 63) {
        if (sc->abort || ld_relaxed(&P.ctrl->abort)) return false;
        if (gtimer() - t0 > P.timeout_ns) {
          record_error(P, kErrTimeout, 4, step);
          sc->abort = 1;
          return false;
        }
      }
    }
    __threadfence_block();
    return true;
  }

  // Every tile is at most g x kc halves of its segment shape, or one attention
  // sub-block of K or V rows; the host sizes the stages to hold both. Checked
  // once here rather than per copy (the copy path is inlined at every issue
  // site): a plan that breaks it copies nothing.
  __device__ bool tiles_fit() const {
    bool fit = kAttnSub * P.dh * 2 <= P.stage_bytes;
    for (int k = 0; k < SK_COUNT; ++k) fit = fit && P.shp[k].g * P.shp[k].kc * 2 <= P.stage_bytes;
    return fit;
  }

  __device__ void run() {
    if (!tiles_fit()) {
      if (lane == 0) record_error(P, kErrDevice, 7, 0);
      sc->abort = 1;
      return;
    }
    bool ok = true;
    unsigned route_round = 0;
    for (step = 0; ok && step < P.n_steps; ++step) {
      for (int l = 0; ok && l < P.L; ++l) {
        ok = issue(dc.at(l, 0), P.shp[SK_QKV]) && issue_attn(l, P.pos0 + step) && issue(dc.at(l, 1), P.shp[SK_O]);
        if (!ok) break;
        if constexpr (!MOE) {
          ok = issue(dc.at(l, 2), P.shp[SK_GU]) && issue(dc.at(l, 3), P.shp[SK_DOWN]);
        } else {
          ok = issue(dc.at(l, 2), P.shp[SK_SGU]);
          if (!ok) break;
          // the routed experts are known only once the consumers have run the router
          ok = wait_route(route_round);
          if (!ok) break;
          int e[kMaxTopK];
          for (int k = 0; k < P.top_k; ++k) e[k] = sc->route_e[route_round % kRouteRing][k];
          ++route_round;
          for (int k = 0; ok && k < P.top_k; ++k) ok = issue(dc.at(l, 4 + e[k]), P.shp[SK_EGU]);
          ok = ok && issue(dc.at(l, 3), P.shp[SK_SDOWN]);
          for (int k = 0; ok && k < P.top_k; ++k) ok = issue(dc.at(l, 4 + P.E + e[k]), P.shp[SK_EDOWN]);
        }
      }
      if (ok && step >= P.lm_from_step) ok = issue(dc.at(P.L, 0), P.shp[SK_LM]);
    }
    // let this lane's last copy land before the CTA may exit
    if (mine > 0) {
      const unsigned n = (mine - 1);  // round of the last tile in this stage
      const unsigned long long t0 = gtimer();
      while (!mbar_test(&sc->full[lane], n & 1u)) {
        if (gtimer() - t0 > P.timeout_ns) break;
      }
    }
  }
};

// ---------------------------------------------------------------- consumer

// One tile: G rows x nch 16-byte chunks, row-major in the stage at shared
// address w_s; the fp32 input slice in the split layout of the vector buffer
// (first halves of the 8-float chunks at x_s, second halves xpb bytes on, so a
// warp's 16-byte loads are contiguous). Lane l takes chunks l, l+32, ...;
// the input chunk is read once and reused for all G rows. Writes the G row
// partial sums to part[pidx0 + r * pstride].
template <int G>
__device__ __forceinline__ void tile_gemv(uint32_t w_s, uint32_t x_s, uint32_t xpb, int nch, int lane, float* part,
                                          int pidx0, int pstride, uint64_t* empty) {
  float acc[G];
#pragma unroll
  for (int r = 0; r < G; ++r) acc[r] = 0.f;
#pragma unroll 2
  for (int c = lane; c < nch; c += 32) {
    const float4 a = lds_f4(x_s + c * 16);
    const float4 b = lds_f4(x_s + xpb + c * 16);
#pragma unroll
    for (int r = 0; r < G; ++r) acc[r] = dot8(lds_u4(w_s + (uint32_t)(r * nch + c) * 16u), a, b, acc[r]);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(empty);  // stage free for the next copy
#pragma unroll
  for (int r = 0; r < G; ++r) {
    const float v = warp_sum(acc[r]);
    if (lane == r) part[pidx0 + r * pstride] = v;
  }
}

// Tile of g <= GM rows x 32*CPL chunks (rows past g are zeroed): the lane's
// share is in registers (wr), then two accumulators per row, and one
// butterfly turns the rows' lane partials into lane r holding row r's sum.
template <int GM, int CPL>
__device__ __forceinline__ void tile_rows_compute(const uint4 (&wr)[GM][CPL], uint32_t x_s, uint32_t xpb, int lane,
                                                  float* part, int pidx0, int pstride, int g) {
  constexpr int NP = GM <= 8 ? 8 : 16;
  float acc[GM][2];
#pragma unroll
  for (int r = 0; r < GM; ++r) acc[r][0] = acc[r][1] = 0.f;
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    const uint32_t xa = x_s + (uint32_t)(lane + 32 * k) * 16u;
    const float4 a = lds_f4(xa), b = lds_f4(xa + xpb);
#pragma unroll
    for (int r = 0; r < GM; ++r) acc[r][k & 1] = dot8(wr[r][k], a, b, acc[r][k & 1]);
  }
  float v[NP];
#pragma unroll
  for (int r = 0; r < NP; ++r) v[r] = r < GM ? acc[r][0] + acc[r][1] : 0.f;
  const float t = transpose_reduce<NP>(v, lane);
  if (lane < g) part[pidx0 + lane * pstride] = t;
}

// The tile from its ring stage: copy the lane's share out and release the
// stage at once.
template <int GM, int CPL>
__device__ __forceinline__ void tile_gemv_rows(uint32_t w_s, uint32_t x_s, uint32_t xpb, int lane, float* part,
                                               int pidx0, int pstride, uint64_t* empty, int g) {
  constexpr int nch = CPL * 32;
  uint4 wr[GM][CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k)
#pragma unroll
    for (int r = 0; r < GM; ++r)
      wr[r][k] = r < g ? lds_u4(w_s + (uint32_t)(r * nch + lane + 32 * k) * 16u) : make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
  if (lane == 0) mbar_arrive(empty);
  tile_rows_compute<GM, CPL>(wr, x_s, xpb, lane, part, pidx0, pstride, g);
}

// K/V row slice of one lane (DPL fp16 head dims) from shared memory.
template <int DPL>
__device__ __forceinline__ uint2 lds_kv(uint32_t a) {
  uint2 r = make_uint2(0u, 0u);
  if constexpr (DPL == 4) asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
  else asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r.x) : "r"(a));
  return r;
}
template <int DPL>
__device__ __forceinline__ void kv_to_f32(uint2 r, float* f) {
  const float2 a = h2f2(r.x);
  f[0] = a.x;
  f[1] = a.y;
  if constexpr (DPL == 4) {
    const float2 b = h2f2(r.y);
    f[2] = b.x;
    f[3] = b.y;
  }
}
// This lane's share of q . k for one row.
template <int DPL>
__device__ __forceinline__ float qk_partial(const float* q, uint2 r) {
  float f[DPL];
  kv_to_f32<DPL>(r, f);
  float t = q[0] * f[0];
#pragma unroll
  for (int e = 1; e < DPL; ++e) t = fmaf(q[e], f[e], t);
  return t;
}

// HD: head_dim (64 or 128); MOE: routed-expert FFN. One kernel is compiled
// per combination, so each model runs only its own code.
template <int HD, bool MOE>
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

  const DescCache dc;

  __device__ Consumer(const Params& p, SmemCtl* s, float* pa, float* v, unsigned char* r, const DescCache& d)
      : P(p), sc(s), part(pa), vec(v), ring(r), tid(threadIdx.x), warp(threadIdx.x >> 5),
        lane(threadIdx.x & 31), dc(d) {}


  // Phase trace (KIE_TRACE builds): per CTA and step, one record of four
  // %globaltimer stamps per phase -- phase start (before its input wait),
  // input ready, tiles (or attention) done, epilogue done -- and a last record
  // for the step barrier (arrival, then release three times). Thread 0 writes
  // the stamps; it passes every consumer barrier, so they are CTA-wide times.
  __device__ __forceinline__ int trace_recs_per_step() const { return 5 * P.L + 2; }
  __device__ __forceinline__ void tstamp(int ph, int i) {
#ifdef KIE_TRACE
    if (P.trace && tid == 0) {
      const int rec = step * trace_recs_per_step() + ph;
      if (rec < P.trace_cap) P.trace[((size_t)blockIdx.x * P.trace_cap + rec) * 4 + i] = gtimer();
    }
#else
    (void)ph;
    (void)i;
#endif
  }

  __device__ __forceinline__ unsigned epoch(int l) const { return 1u + (unsigned)step * (unsigned)(P.L + 1) + (unsigned)l; }

  // Four flagged words at p (16-byte aligned) once they all carry epoch ep.
  // Bounded: on abort or deadline it flags the CTA and returns zeros.
  __device__ __forceinline__ float4 wait4(const unsigned long long* p, unsigned ep) {
    unsigned long long a, b, c, d;
    ld_flag2(p, a, b);
    ld_flag2(p + 2, c, d);
    if (fepoch(a) != ep || fepoch(b) != ep || fepoch(c) != ep || fepoch(d) != ep) {
      const unsigned long long t0 = gtimer();
      for (unsigned it = 1;; ++it) {
        ld_flag2(p, a, b);
        ld_flag2(p + 2, c, d);
        if (fepoch(a) == ep && fepoch(b) == ep && fepoch(c) == ep && fepoch(d) == ep) break;
        if ((it & 31) == 0) {
          if (sc->abort || ld_relaxed(&P.ctrl->abort)) {
            sc->abort = 1;
            return make_float4(0.f, 0.f, 0.f, 0.f);
          }
          if (gtimer() - t0 > P.timeout_ns) {
            record_error(P, kErrTimeout, 6, step);
            sc->abort = 1;
            return make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
    }
    return make_float4(fval(a), fval(b), fval(c), fval(d));
  }

  // The vector buffer holds an input vector split by halves of its 8-float
  // chunks: element i of chunk c (i < 4) at vec[4c + i], element 4 + i at
  // vec[xplane + 4c + i]. xv(i) is where the 4 elements from i (i % 4 == 0) go.
  __device__ __forceinline__ float* xv(int i) const {
    return vec + ((i & 4) ? P.xplane : 0) + ((i >> 3) << 2);
  }

  // The flagged words src[i..i+4) for the kLoadBatch groups i = base + b *
  // kConsumerThreads * 4 (those below n), once they carry epoch ep, into v.
  // Every lane of the warp must call it together (warp-wide votes decide when
  // the warp stops polling).
  // All of the batch's loads are issued before any epoch is checked, and the
  // groups still stale are re-polled together, so a thread waits about one L2
  // round trip per batch instead of one per group. Bounded: on abort or
  // deadline it flags the CTA and leaves zeros. Four groups a thread (a
  // 3584-float vector in one batch) measured fastest among 2, 3, 4, 6 and 8.
  static constexpr int kLoadBatch = 4;
  __device__ __forceinline__ void fetch_batch(const unsigned long long* src, unsigned ep, int n, int base,
                                              float4 (&v)[kLoadBatch]) {
    unsigned long long w[kLoadBatch][4];
#pragma unroll
    for (int b = 0; b < kLoadBatch; ++b) {
      const int i = base + b * kConsumerThreads * 4;
      w[b][0] = w[b][1] = w[b][2] = w[b][3] = (unsigned long long)ep << 32;
      if (i < n) {
        ld_flag2(src + i, w[b][0], w[b][1]);
        ld_flag2(src + i + 2, w[b][2], w[b][3]);
      }
    }
    unsigned long long t0 = 0;
    // the warp loops together (warp-uniform exit and give-up)
    for (unsigned it = 0;; ++it) {
      bool stale = false;
#pragma unroll
      for (int b = 0; b < kLoadBatch; ++b) {
        const int i = base + b * kConsumerThreads * 4;
        if (fepoch(w[b][0]) != ep || fepoch(w[b][1]) != ep || fepoch(w[b][2]) != ep || fepoch(w[b][3]) != ep) {
          stale = true;
          ld_flag2(src + i, w[b][0], w[b][1]);
          ld_flag2(src + i + 2, w[b][2], w[b][3]);
        }
      }
      if (!__any_sync(0xffffffffu, stale)) break;
      if (it == 0) {
        t0 = gtimer();
      } else if ((it & 31) == 0) {
        bool give_up = false;
        if (sc->abort || ld_relaxed(&P.ctrl->abort)) {
          give_up = true;
        } else if (gtimer() - t0 > P.timeout_ns) {
          record_error(P, kErrTimeout, 6, step);
          give_up = true;
        }
        if (__any_sync(0xffffffffu, give_up)) {
          sc->abort = 1;
#pragma unroll
          for (int b = 0; b < kLoadBatch; ++b) v[b] = make_float4(0.f, 0.f, 0.f, 0.f);
          return;
        }
      }
    }
#pragma unroll
    for (int b = 0; b < kLoadBatch; ++b) v[b] = make_float4(fval(w[b][0]), fval(w[b][1]), fval(w[b][2]), fval(w[b][3]));
  }

  // vec = the flagged vector src[0..n) of epoch ep (n a multiple of 8), once
  // its producers have written it
  __device__ void load_vec(const unsigned long long* src, unsigned ep, int n) {
    // warp-uniform trip count: fetch_batch's warp-wide votes need every lane
    // (lanes past n hold only groups that are already complete)
    for (int base0 = warp * 128; base0 < n; base0 += kConsumerThreads * 4 * kLoadBatch) {
      const int base = base0 + lane * 4;
      float4 v[kLoadBatch];
      fetch_batch(src, ep, n, base, v);
#pragma unroll
      for (int b = 0; b < kLoadBatch; ++b) {
        const int i = base + b * kConsumerThreads * 4;
        if (i < n) *reinterpret_cast<float4*>(xv(i)) = v[b];
      }
    }
    cbar();
  }

  // Start copying the next RMSNorm gain into the shared gain buffer
  // (cp.async, no registers held); load_norm waits for it. Each thread copies
  // the four gains of exactly the elements it will scale in load_norm, so
  // waiting for its own copies is enough. Issued right after the previous
  // load_norm, so the copy overlaps a whole phase.
  __device__ void prefetch_gain(const __half* g) {
    const uint32_t gb = su32(vec + P.gbuf_off);
    for (int i = tid * 4; i < P.d; i += kConsumerThreads * 4)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(gb + i * 2), "l"(g + i) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  // vec = gain * x, with x either the flagged residual stream of epoch ep or
  // an fp16 embedding row (the gain was prefetched by prefetch_gain). RMSNorm's
  // factor 1/sqrt(mean(x^2) + eps) is a scalar, so it is applied to the GEMV
  // outputs in the epilogue (norm_scale) instead of to x: the tiles start
  // right after the load, and this CTA's sum of squares travels through the
  // one barrier the load needs anyway.
  __device__ void load_norm(const unsigned long long* srcf, unsigned ep, const __half* srch, int n) {
    asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's gain copies
    const __half* gb = reinterpret_cast<const __half*>(vec + P.gbuf_off);
    float ss = 0.f;
    // warp-uniform trip count, as in load_vec
    for (int base0 = warp * 128; base0 < n; base0 += kConsumerThreads * 4 * kLoadBatch) {
      const int base = base0 + lane * 4;
      float4 v[kLoadBatch];
      if (srcf) {
        fetch_batch(srcf, ep, n, base, v);
      } else {
#pragma unroll
        for (int b = 0; b < kLoadBatch; ++b) {
          const int i = base + b * kConsumerThreads * 4;
          v[b] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < n) {
            const uint2 raw = *reinterpret_cast<const uint2*>(srch + i);
            const float2 lo = h2f2(raw.x), hi = h2f2(raw.y);
            v[b] = make_float4(lo.x, lo.y, hi.x, hi.y);
          }
        }
      }
#pragma unroll
      for (int b = 0; b < kLoadBatch; ++b) {
        const int i = base + b * kConsumerThreads * 4;
        if (i < n) {
          const float4 x = v[b];
          ss = fmaf(x.x, x.x, ss);
          ss = fmaf(x.y, x.y, ss);
          ss = fmaf(x.z, x.z, ss);
          ss = fmaf(x.w, x.w, ss);
          const uint2 g = *reinterpret_cast<const uint2*>(gb + i);
          const float2 g0 = h2f2(g.x), g1 = h2f2(g.y);
          *reinterpret_cast<float4*>(xv(i)) = make_float4(x.x * g0.x, x.y * g0.y, x.z * g1.x, x.w * g1.y);
        }
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) sc->ssq[warp] = ss;
    cbar();
  }

  // 1/sqrt(mean(x^2) + eps) of the vector the last load_norm read
  __device__ __forceinline__ float norm_scale() const {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) t += sc->ssq[w];
    return 1.0f / sqrtf(t / (float)P.d + P.eps);
  }

  // The output projection's input wait (the attention chain) is the longest
  // wait of a layer, and HBM is mostly idle during it: the ring already holds
  // the output projection's tiles and the first gate/up tiles. Meanwhile the
  // consumers prefetch into L2 kGuPrefetch bytes of this CTA's gate/up tiles
  // from the (ring stages / 2)-th on, so the gate/up phase reads them from L2.
  // Measured on the 2.2B model: 192 KB from tile 7 best (from tile 10 the
  // same; from tile 4 or 14, or 128, 256 and 384 KB, less or slower, as were
  // prefetches in the other phases' waits).
  static constexpr int kGuPrefetch = 192 * 1024;
  __device__ __forceinline__ void prefetch_gate_up(int l) {
    const SegDesc& gu = dc.at(l, 2);
    const SegShape& gs = P.shp[SK_GU];
    const unsigned long long seg = (unsigned long long)gu.nrows * gs.K * 2ull;
    const unsigned long long a0 =
        (unsigned long long)(P.n_stages / 2) * gs.g * gs.kc * 2ull + (unsigned long long)tid * 4096ull;
    if (tid < kGuPrefetch / 4096 && a0 < seg) {
      const unsigned sz = (unsigned)min(4096ull, seg - a0);  // multiples of 16 B at 16-byte aligned tape offsets
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(P.tape + gu.off + a0), "r"(sz) : "memory");
    }
  }

  // Consume one segment's tiles; partial sums land in part[pbase + row*pstride + kjbase + kj].
  __device__ void run_segment(const SegDesc& sd, const SegShape& sh, const float* vseg, int pbase,
                              int pstride, int kjbase) {
    const int ngroups = (sd.nrows + sh.g - 1) / sh.g;
    const int ntiles = ngroups * sh.nk;
    const int ns = P.n_stages;
    const int nch = sh.kc / 8;
    // Tile t (ring position) always goes to warp t % kConsumerWarps, and the
    // stage count is a multiple of kConsumerWarps, so every stage is only ever
    // used by one warp, in order: its parity waits can never see a phase two
    // rounds old.
    const int first = (int)((warp + kConsumerWarps - (int)(tbase % kConsumerWarps)) % kConsumerWarps);
    // stage, parity and (row group, column block) of this warp's tiles,
    // advanced without divisions: each step is kConsumerWarps tiles on
    const unsigned t0 = tbase + (unsigned)first;
    int s = (int)(t0 % (unsigned)ns);
    unsigned par = (t0 / (unsigned)ns) & 1u;
    int gi = first / sh.nk, kj = first - gi * sh.nk;
    const int dg = kConsumerWarps / sh.nk, dk = kConsumerWarps - dg * sh.nk;
    for (int i = first; i < ntiles; i += kConsumerWarps) {
      if (sc->abort) break;
      if (!wait_bar(P, sc, &sc->full[s], par, 2, step)) break;
      const int gp = min(sh.g, sd.nrows - gi * sh.g);
      const uint32_t w = su32(ring) + (uint32_t)(s * P.stage_bytes);
      const uint32_t xs = su32(vseg) + (uint32_t)(kj * sh.kc) * 2u;
      const uint32_t xpb = (uint32_t)P.xplane * 4u;
      const int p0 = pbase + gi * sh.g * pstride + kjbase + kj;
      uint64_t* em = &sc->empty[s];
      bool done = true;
      if (nch == 64 && gp <= 13) tile_gemv_rows<13, 2>(w, xs, xpb, lane, part, p0, pstride, em, gp);
      else if (nch == 96 && gp <= 8) tile_gemv_rows<8, 3>(w, xs, xpb, lane, part, p0, pstride, em, gp);
      else done = false;
      if (!done) {
        switch (gp) {
          case 1: tile_gemv<1>(w, xs, xpb, nch, lane, part, p0, pstride, em); break;
          case 2: tile_gemv<2>(w, xs, xpb, nch, lane, part, p0, pstride, em); break;
          case 3: tile_gemv<3>(w, xs, xpb, nch, lane, part, p0, pstride, em); break;
          case 4: tile_gemv<4>(w, xs, xpb, nch, lane, part, p0, pstride, em); break;
          case 5: tile_gemv<5>(w, xs, xpb, nch, lane, part, p0, pstride, em); break;
          case 6: tile_gemv<6>(w, xs, xpb, nch, lane, part, p0, pstride, em); break;
          case 7: tile_gemv<7>(w, xs, xpb, nch, lane, part, p0, pstride, em); break;
          default: tile_gemv<8>(w, xs, xpb, nch, lane, part, p0, pstride, em); break;
        }
      }
      s += kConsumerWarps;
      if (s >= ns) {
        s -= ns;
        par ^= 1u;
      }
      kj += dk;
      gi += dg;
      if (kj >= sh.nk) {
        kj -= sh.nk;
        ++gi;
      }
    }
    tbase += ntiles;
  }

  __device__ float row_sum(int r, int stride) const {
    float y = 0.f;
    for (int k = 0; k < stride; ++k) y += part[r * stride + k];
    return y;
  }

  // Grid-wide barrier, once per step (see run). Returns false if the run aborted.
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
        // the consumer barrier above orders this CTA's writes before thread 0's
        // release; the release-add publishes them at GPU scope
        if (!skip) red_release_add(&P.ctrl->arrive, 1u);
        const unsigned target = (k + 1) * gridDim.x;
        const unsigned long long t0 = gtimer();
        unsigned it = 0;
        while (ld_relaxed(&P.ctrl->arrive) < target) {
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
        asm volatile("fence.acq_rel.gpu;" ::: "memory");  // acquire the other CTAs' writes
      }
#ifdef KIE_TRACE
      if (P.trace) {
        const int rec = step * trace_recs_per_step() + trace_recs_per_step() - 1;
        if (rec < P.trace_cap) {
          unsigned long long* tr = P.trace + ((size_t)blockIdx.x * P.trace_cap + rec) * 4;
          const unsigned long long tb = gtimer();
          tr[0] = ta;
          tr[1] = tb;
          tr[2] = tb;
          tr[3] = tb;
        }
      }
#else
      if (P.trace && (int)k < P.trace_cap) {
        unsigned long long* tr = P.trace + ((size_t)blockIdx.x * P.trace_cap + k) * 2;
        tr[0] = ta;
        tr[1] = gtimer();
      }
#endif
      sc->abort = ab;
    }
    return !cbar_any(sc->abort != 0);
  }

  // One warp's share of one attention unit for a KV group of NH query heads:
  // its sub-range [wj0, wj1) in 32-position sub-blocks whose K and V tiles come
  // through the ring, with online softmax; the (max, sum, acc) partials of
  // each head go to wp. NH is a template parameter so every head loop is
  // unrolled exactly, keeping the code small.
  template <int DH, int NH>
  __device__ void attn_warp(const AttnPlan& ap, int uo, int vs, int wj0, int wj1, int pos, uint2 kpos,
                            uint2 vpos, float* qs, float* wp, float* sbuf) {
    constexpr int DPL = DH / 32;
    constexpr int WS = DH + 4;
    const int ns = P.n_stages;
    const uint32_t ring_s = su32(ring);
    const uint32_t ssm = su32(sbuf) + (uint32_t)(warp * kMaxHeadsPerGroup * kAttnSub) * 4u;
    const uint32_t qsa = su32(qs) + (uint32_t)(lane * DPL) * 4u;
    float m[NH], ls[NH], acc[NH][DPL], acc2[NH][DPL];
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      m[hh] = -INFINITY;
      ls[hh] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[hh][e] = acc2[hh][e] = 0.f;
    }
    for (int b = 0; b < ap.nsb; ++b) {
      const unsigned tK = tbase + (unsigned)((uo * ap.nsb + b) * kAttnTilesPerRound + vs);
      const unsigned tV = tK + kConsumerWarps;
      const int sK = (int)(tK % ns), sV = (int)(tV % ns);
      const int jb = wj0 + b * kAttnSub;
      const int nj = max(0, min(kAttnSub, wj1 - jb));                  // valid keys in the sub-block
      const int nsm = max(0, min(min(jb + kAttnSub, wj1), pos) - jb);  // of which in the tile
      const bool valid = lane < nj;
      if (!wait_bar(P, sc, &sc->full[sK], (tK / ns) & 1u, 2, step)) sc->abort = 1;
      const bool work = nj > 0 && !sc->abort;
      if (work) {
        const uint32_t kt = ring_s + (uint32_t)(sK * P.stage_bytes) + (uint32_t)(lane * DPL * 2);
#pragma unroll 1
        for (int hh = 0; hh < NH; ++hh) {
          float q[DPL];
#pragma unroll
          for (int e = 0; e < DPL; ++e) q[e] = lds_f32(qsa + (uint32_t)(hh * DH + e) * 4u);
          // All 32 rows of the stage are read; rows past the tile hold stale
          // data whose scores only reach their own (masked) position.
          float part[kAttnSub];
#pragma unroll
          for (int jj = 0; jj < kAttnSub; ++jj) part[jj] = qk_partial<DPL>(q, lds_kv<DPL>(kt + jj * DH * 2));
          float a = transpose_reduce32(part, lane);
          if (nsm < nj) {  // this token's own row, position nsm of the sub-block
            const float own = warp_sum(qk_partial<DPL>(q, kpos));
            if (lane == nsm) a = own;
          }
          sts_f32(ssm + (uint32_t)(hh * kAttnSub + lane) * 4u, valid ? a : -INFINITY);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc->empty[sK]);
      if (!wait_bar(P, sc, &sc->full[sV], (tV / ns) & 1u, 2, step)) sc->abort = 1;
      if (work && !sc->abort) {
        float p[NH];
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          const float sv = lds_f32(ssm + (uint32_t)(hh * kAttnSub + lane) * 4u);
          const float mn = fmaxf(m[hh], warp_max(sv));
          p[hh] = valid ? expf(sv - mn) : 0.f;
          const float corr = expf(m[hh] - mn);
          ls[hh] = ls[hh] * corr + warp_sum(p[hh]);
#pragma unroll
          for (int e = 0; e < DPL; ++e) {
            acc[hh][e] *= corr;
            acc2[hh][e] *= corr;
          }
          m[hh] = mn;
        }
        const uint32_t vt = ring_s + (uint32_t)(sV * P.stage_bytes) + (uint32_t)(lane * DPL * 2);
        // p of every position to shared memory (the score slots), read back
        // four at a time as broadcasts; all 32 rows of the V stage are
        // loaded at once and rows past the tile are masked out by select
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) sts_f32(ssm + (uint32_t)(hh * kAttnSub + lane) * 4u, p[hh]);
        __syncwarp();
#pragma unroll
        for (int j4 = 0; j4 < kAttnSub; j4 += 4) {
          float4 pv[NH];
#pragma unroll
          for (int hh = 0; hh < NH; ++hh) pv[hh] = lds_f4(ssm + (uint32_t)(hh * kAttnSub + j4) * 4u);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = j4 + u;
            float f[DPL];
            kv_to_f32<DPL>(lds_kv<DPL>(vt + j * DH * 2), f);
            const bool in = j < nsm;
#pragma unroll
            for (int e = 0; e < DPL; ++e) f[e] = in ? f[e] : 0.f;
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
              const float pj = u == 0 ? pv[hh].x : u == 1 ? pv[hh].y : u == 2 ? pv[hh].z : pv[hh].w;
#pragma unroll
              for (int e = 0; e < DPL; ++e) {
                if (u & 1) acc2[hh][e] = fmaf(pj, f[e], acc2[hh][e]);
                else acc[hh][e] = fmaf(pj, f[e], acc[hh][e]);
              }
            }
          }
        }
        if (nsm < nj) {  // this token's own row
          float fv[DPL];
          kv_to_f32<DPL>(vpos, fv);
#pragma unroll
          for (int hh = 0; hh < NH; ++hh) {
            const float pv = __shfl_sync(0xffffffffu, p[hh], nsm);
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[hh][e] = fmaf(pv, fv[e], acc[hh][e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc->empty[sV]);
    }
    // partials -> shared memory, in the slot of this warp's sub-range (not of
    // the warp: the warp <-> sub-range map depends on the ring position, and
    // merging in sub-range order keeps results independent of launch history).
    // An empty range gives m = -inf, l = 0.
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      float* pb = wp + (vs * kMaxHeadsPerGroup + hh) * WS;
      if (lane == 0) {
        pb[0] = m[hh];
        pb[1] = ls[hh];
      }
#pragma unroll
      for (int e = 0; e < DPL; ++e) pb[4 + lane * DPL + e] = acc[hh][e] + acc2[hh][e];
    }
  }

  // ---- attention over the KV cache (q already rotated and scaled; this
  // token's k/v appended by the q/k/v epilogue). K and V rows arrive through
  // the ring (see attn_plan); each warp handles one sub-range of each of the
  // CTA's units, lanes over head dims for both q.k (butterfly transpose-reduce
  // of 32 positions) and the V sum. The warps' (max, sum, acc) partials are
  // merged in shared memory; a head split into chunks over several CTAs is
  // finished by the CTA of its chunk 0 from the flagged chunk records.
  // Trace stamps of the phase (KIE_TRACE builds): input = q and this token's
  // k/v of the first unit arrived, tiles = every unit's sub-ranges done and
  // merged in the CTA, epilogue (by the caller) = cross-CTA chunk merges done.
  template <int DH>
  __device__ void attention(int l, int pos, int ph) {
    constexpr int DPL = DH / 32;   // head dims per lane
    constexpr int WS = DH + 4;     // partial record: m, l, pad, pad, acc[DH]
    const int hk = P.hk, hq = P.hq, G = gridDim.x;
    const AttnPlan ap = attn_plan(pos, hk, hq, G);
    const int nu = attn_units_of(ap, blockIdx.x, G);
    const int vs = (int)((warp + kConsumerWarps - (int)(tbase % kConsumerWarps)) % kConsumerWarps);
    float* qs = vec;                                              // [nh][DH]
    float* wp = vec + kMaxHeadsPerGroup * DH;                     // [warp][hh][WS]
    float* sbuf = wp + kConsumerWarps * kMaxHeadsPerGroup * WS;   // [warp][hh][32] scores
    const uint32_t ring_s = su32(ring);
    for (int uo = 0; uo < nu; ++uo) {
      const int u = blockIdx.x + uo * G;
      const AttnUnit au = attn_unit(ap, u, hk, hq);
      const int g = au.g, ch = au.ch, h_lo = au.h_lo, nh = au.nh;
      const int j0 = ch * ap.per, j1 = min(ap.T, j0 + ap.per);
      const int wj0 = j0 + vs * ap.pw, wj1 = min(j1, wj0 + ap.pw);
      // q of this group's heads and this token's own k/v row (not in the ring)
      // come flagged from the q/k/v epilogues that produced them
      const unsigned ep = epoch(l);
      for (int i = tid * 4; i < nh * DH; i += kConsumerThreads * 4)
        *reinterpret_cast<float4*>(qs + i) = wait4(P.fq + (size_t)h_lo * DH + i, ep);
      uint2 kpos = make_uint2(0u, 0u), vpos = make_uint2(0u, 0u);
      if (wj0 <= pos && pos < wj1) {
        const unsigned long long* kr = P.fq + (size_t)(hq + g) * DH + lane * DPL;
        const unsigned long long* vr = P.fq + (size_t)(hq + hk + g) * DH + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 kf = wait4(kr, ep), vf = wait4(vr, ep);
          kpos = make_uint2(f2h2(kf.x, kf.y), f2h2(kf.z, kf.w));
          vpos = make_uint2(f2h2(vf.x, vf.y), f2h2(vf.z, vf.w));
        } else {
          // two dims per lane: the aligned group of four holds this lane's pair
          const float4 kf = wait4(kr - (lane & 1) * 2, ep), vf = wait4(vr - (lane & 1) * 2, ep);
          kpos.x = (lane & 1) ? f2h2(kf.z, kf.w) : f2h2(kf.x, kf.y);
          vpos.x = (lane & 1) ? f2h2(vf.z, vf.w) : f2h2(vf.x, vf.y);
        }
      }
      if (cbar_any(sc->abort != 0)) return;
      if (uo == 0) tstamp(ph, 1);
      switch (nh) {
        case 1: attn_warp<DH, 1>(ap, uo, vs, wj0, wj1, pos, kpos, vpos, qs, wp, sbuf); break;
        case 2: attn_warp<DH, 2>(ap, uo, vs, wj0, wj1, pos, kpos, vpos, qs, wp, sbuf); break;
        case 3: attn_warp<DH, 3>(ap, uo, vs, wj0, wj1, pos, kpos, vpos, qs, wp, sbuf); break;
        default: attn_warp<DH, 4>(ap, uo, vs, wj0, wj1, pos, kpos, vpos, qs, wp, sbuf); break;
      }
      cbar();
      // merge the sub-ranges' partials in sub-range order: warp hh merges head hh
      if (warp < nh) {
        const int hh = warp;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, wp[(w * kMaxHeadsPerGroup + hh) * WS]);
        float Ls = 0.f, a[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) a[e] = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float* pb = wp + (w * kMaxHeadsPerGroup + hh) * WS;
          const float sc_w = expf(pb[0] - M);
          Ls = fmaf(sc_w, pb[1], Ls);
#pragma unroll
          for (int e = 0; e < DPL; ++e) a[e] = fmaf(sc_w, pb[4 + lane * DPL + e], a[e]);
        }
        const int h = h_lo + hh;
        if (ap.nchk == 1) {
          const float inv = 1.0f / Ls;
          unsigned long long* ob = P.fo + (size_t)h * DH + lane * DPL;
#pragma unroll
          for (int e = 0; e < DPL; e += 2) st_flag2(ob + e, a[e] * inv, a[e + 1] * inv, epoch(l));
        } else {
          // this chunk's record of head h, flagged: (max, sum) then acc[DH]
          unsigned long long* gb = P.apart + ((size_t)h * P.max_chunks + ch) * WS;
          if (lane == 0) st_flag2(gb, M, Ls, epoch(l));
#pragma unroll
          for (int e = 0; e < DPL; e += 2) st_flag2(gb + 4 + lane * DPL + e, a[e], a[e + 1], epoch(l));
        }
      }
      cbar();  // qs / wp are reused by the next unit
    }
    if (nu == 0) tstamp(ph, 1);
    tstamp(ph, 2);
    // A KV head split into chunks is finished by the CTA of its chunk 0. That
    // CTA merges only after it has published the records of all its own units,
    // so no CTA waits for a record that one of its later units would produce.
    if (ap.nchk > 1) {
      for (int uo = 0; uo < nu; ++uo) {
        const int u = blockIdx.x + uo * G;
        const AttnUnit au = attn_unit(ap, u, hk, hq);
        if (au.ch != 0) continue;
        if (warp < au.nh) merge_chunks<DH>(au.h_lo + warp, ap.nchk, epoch(l));
      }
    }
    tbase += (unsigned)(nu * ap.nsb * kAttnTilesPerRound);
  }

  // Merge the nchk chunk records of query head h into its attention output, in
  // chunk order with a running (max, sum, acc) rescaled per chunk. One warp;
  // lane l owns head dims l*DPL .. l*DPL + DPL - 1. The flagged words of a
  // batch of chunks are all loaded before any epoch is checked and the stale
  // ones re-polled together (one L2 round trip once the last chunk is out).
  template <int DH>
  __device__ void merge_chunks(int h, int nchk, unsigned ep) {
    constexpr int DPL = DH / 32, WS = DH + 4, B = 8, NW = 2 + DPL;
    const unsigned long long* hb = P.apart + (size_t)h * P.max_chunks * WS;
    float M = -INFINITY, Ls = 0.f, acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
    for (int c0 = 0; c0 < nchk; c0 += B) {
      unsigned long long w[B][NW];
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const unsigned long long* cb = hb + (size_t)(c0 + b) * WS;
#pragma unroll
        for (int i = 0; i < NW; ++i) w[b][i] = (unsigned long long)ep << 32;
        if (c0 + b < nchk) {
          ld_flag2(cb, w[b][0], w[b][1]);
#pragma unroll
          for (int e = 0; e < DPL; e += 2) ld_flag2(cb + 4 + lane * DPL + e, w[b][2 + e], w[b][3 + e]);
        }
      }
      unsigned long long t0 = 0;
      for (unsigned it = 0;; ++it) {
        bool stale = false;
#pragma unroll
        for (int b = 0; b < B; ++b) {
          bool st = false;
#pragma unroll
          for (int i = 0; i < NW; ++i) st |= fepoch(w[b][i]) != ep;
          if (st) {
            stale = true;
            const unsigned long long* cb = hb + (size_t)(c0 + b) * WS;
            ld_flag2(cb, w[b][0], w[b][1]);
#pragma unroll
            for (int e = 0; e < DPL; e += 2) ld_flag2(cb + 4 + lane * DPL + e, w[b][2 + e], w[b][3 + e]);
          }
        }
        if (!stale) break;
        if (it == 0) {
          t0 = gtimer();
        } else if ((it & 31) == 0) {
          if (sc->abort || ld_relaxed(&P.ctrl->abort)) {
            sc->abort = 1;
            return;
          }
          if (gtimer() - t0 > P.timeout_ns) {
            record_error(P, kErrTimeout, 6, step);
            sc->abort = 1;
            return;
          }
        }
      }
#pragma unroll
      for (int b = 0; b < B; ++b) {
        if (c0 + b >= nchk) break;
        const float m = fval(w[b][0]), l = fval(w[b][1]);
        const float Mn = fmaxf(M, m);
        const float so = expf(M - Mn), sn = expf(m - Mn);
        Ls = Ls * so + l * sn;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = acc[e] * so + fval(w[b][2 + e]) * sn;
        M = Mn;
      }
    }
    const float inv = 1.0f / Ls;
    unsigned long long* ob = P.fo + (size_t)h * DH + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; e += 2) st_flag2(ob + e, acc[e] * inv, acc[e + 1] * inv, ep);
  }

  __device__ void attention_dispatch(int l, int pos, int ph) { attention<HD>(l, pos, ph); }

  // Copy the RoPE coefficients of this CTA's first kRopeStage q/k row pairs at
  // position pos into shared memory (cp.async; load_norm's wait covers it).
  // The thread that copies pair j is the one whose epilogue rotates it.
  __device__ void stage_rope(const SegDesc& sd, int pos) {
    const int dh = P.dh, npairs = min(sd.nrows / 2, kRopeStage);
    const float2* rp = P.rope + (size_t)pos * (dh / 2);
    for (int j = tid; j < npairs; j += kConsumerThreads) {
      const int r = sd.row0 + 2 * j;
      const int H = r / dh, pi = (r - H * dh) / 2;
      if (H < P.hq + P.hk)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(su32(&sc->rcs[j])), "l"(rp + pi) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  // q/k/v epilogue. The q/k/v rows are packed so that every CTA owns whole
  // RoPE pairs (dims i and i + dh/2 of one head are adjacent virtual rows), so
  // RoPE is applied here: q is rotated and pre-scaled by 1/sqrt(dh), k is
  // rotated and appended (fp16) to the KV cache at `pos`, v is appended as is;
  // q and the fp16-rounded k and v are also published flagged for this step's
  // attention.
  __device__ void epi_qkv(const SegDesc& sd, int stride, int l, int pos) {
    const int dh = P.dh, half = P.dh / 2, hq = P.hq, hk = P.hk;
    const float2* rp = P.rope + (size_t)pos * half;
    const float scale = 1.0f / sqrtf((float)dh);
    const float inv = norm_scale();
    const unsigned ep = epoch(l);
    for (int j = tid; j < sd.nrows / 2; j += kConsumerThreads) {
      const int r = sd.row0 + 2 * j;
      const int H = r / dh, pi = (r - H * dh) / 2;
      const float ya = row_sum(2 * j, stride) * inv, yb = row_sum(2 * j + 1, stride) * inv;
      if (H < hq + hk) {
        const float2 cs = j < kRopeStage ? sc->rcs[j] : rp[pi];
        const float a = ya * cs.x - yb * cs.y, b = ya * cs.y + yb * cs.x;
        if (H < hq) {
          st_flag(P.fq + (size_t)H * dh + pi, a * scale, ep);
          st_flag(P.fq + (size_t)H * dh + pi + half, b * scale, ep);
        } else {
          __half* k = P.kcache + ((size_t)(l * hk + (H - hq)) * P.max_ctx + pos) * dh;
          const __half ka = __float2half_rn(a), kb = __float2half_rn(b);
          k[pi] = ka;
          k[pi + half] = kb;
          st_flag(P.fq + (size_t)H * dh + pi, __half2float(ka), ep);
          st_flag(P.fq + (size_t)H * dh + pi + half, __half2float(kb), ep);
        }
      } else {
        __half* v = P.vcache + ((size_t)(l * hk + (H - hq - hk)) * P.max_ctx + pos) * dh;
        const __half va = __float2half_rn(ya), vb = __float2half_rn(yb);
        v[pi] = va;
        v[pi + half] = vb;
        st_flag(P.fq + (size_t)H * dh + pi, __half2float(va), ep);
        st_flag(P.fq + (size_t)H * dh + pi + half, __half2float(vb), ep);
      }
    }
    // the cache rows written here are read by TMA (async proxy) in later steps
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }

  // residual epilogue: x[row] = xprev[row] + sum of partials. xprev is this
  // CTA's own copy of its rows (or the embedding row in the first layer).
  // The new rows are published flagged in the residual buffer `which`.
  __device__ void epi_residual(const SegDesc& sd, int stride, const __half* xprev_h, int which, unsigned ep) {
    unsigned long long* fx = P.fx + (size_t)which * P.d;
    for (int r = tid; r < sd.nrows; r += kConsumerThreads) {
      const int row = sd.row0 + r;
      const float xp = xprev_h ? __half2float(xprev_h[row]) : sc->xown[r];
      const float v = xp + row_sum(r, stride);
      sc->xown[r] = v;
      st_flag(fx + row, v, ep);
    }
    if constexpr (MOE) {
      if (which == 0) router_partials(sd, ep);
    }
  }

  // MoE router logit e = (R_e . (g * x)) / rms(x), with x the residual stream
  // after the output projection and g the FFN RMSNorm gain. Both the dot
  // product and the sum of squares split over the residual rows, so every CTA
  // publishes its rows' share of each (flagged, row e of froute for logit e,
  // row E for the squares) and the router needs no GEMV of its own: the
  // FFN-up phase sums the grid's shares (route). The router columns of the
  // rows were staged in shared memory by prefetch_router, and the gain by
  // prefetch_gain.
  __device__ void router_partials(const SegDesc& sd, unsigned ep) {
    asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's gain copies
    cbar();  // every row's x, every thread's gain copies and the staged router columns
    const __half* rs = reinterpret_cast<const __half*>(vec + P.rslice_off);
    const __half* gb = reinterpret_cast<const __half*>(vec + P.gbuf_off);
    const int n = sd.nrows, cap = P.rslice_rows;
    for (int e = warp; e <= P.E; e += kConsumerWarps) {
      float a = 0.f;
      for (int r = lane; r < n; r += 32) {
        const float x = sc->xown[r];
        a = e < P.E ? fmaf(__half2float(rs[e * cap + r]) * __half2float(gb[sd.row0 + r]), x, a) : fmaf(x, x, a);
      }
      a = warp_sum(a);
      if (lane == 0) st_flag(P.froute + (size_t)e * ((gridDim.x + 1) & ~1u) + blockIdx.x, a, ep);
    }
  }

  // Stage layer l's router columns of this CTA's residual rows in shared
  // memory ([E][rslice_rows] fp16), during the output projection's input wait.
  __device__ void prefetch_router(int l, const SegDesc& sd) {
    __half* rs = reinterpret_cast<__half*>(vec + P.rslice_off);
    const __half* R = P.router + (size_t)l * P.E * P.d + sd.row0;
    const int n = sd.nrows, cap = P.rslice_rows;
    for (int i = tid; i < P.E * n; i += kConsumerThreads) {
      const int e = i / n, r = i - e * n;
      rs[e * cap + r] = R[(size_t)e * P.d + r];
    }
  }

  // SwiGLU epilogue over interleaved (gate, up) rows: h[hoff + row0/2 + j] = w * silu(g) * u
  __device__ void epi_swiglu(const SegDesc& sd, int pbase, int stride, int hoff, float w, unsigned ep) {
    const int npairs = sd.nrows / 2;
    const float inv = norm_scale();
    for (int j = tid; j < npairs; j += kConsumerThreads) {
      float yg = 0.f, yu = 0.f;
      for (int k = 0; k < stride; ++k) {
        yg += part[pbase + (2 * j) * stride + k];
        yu += part[pbase + (2 * j + 1) * stride + k];
      }
      yg *= inv;
      yu *= inv;
      st_flag(P.fh + hoff + sd.row0 / 2 + j, w * silu(yg) * yu, ep);
    }
  }

  // MoE routing, decided identically by every CTA: the logits are the sums of
  // the grid's flagged router partials (router_partials), added in one fixed
  // order (warp e % 7 sums row e, each lane its CTAs 2 lane + 64 k, k < 3,
  // then a butterfly), so every CTA takes the same decision from the same
  // words. Rows are polled kRouteRows at a time, all loads issued first.
  static constexpr int kRouteRows = 4;
  __device__ void route(int l) {
    const int G = gridDim.x, E = P.E, gp = (G + 1) & ~1;  // rows padded to pairs
    const unsigned ep = epoch(l);
    // warp-uniform trip count: the polls' votes need every lane
    for (int e0 = warp; e0 <= E; e0 += kConsumerWarps * kRouteRows) {
      unsigned long long w[kRouteRows][3][2];
#pragma unroll
      for (int b = 0; b < kRouteRows; ++b) {
        const int e = e0 + b * kConsumerWarps;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          const int c = 2 * lane + 64 * k;
          w[b][k][0] = w[b][k][1] = fpack(0.f, ep);
          if (e <= E && c < G) {
            const unsigned long long* src = P.froute + (size_t)e * gp + c;
            if (c + 1 < G) ld_flag2(src, w[b][k][0], w[b][k][1]);
            else w[b][k][0] = ld_flag1(src);
          }
        }
      }
      unsigned long long t0 = 0;
      for (unsigned it = 0;; ++it) {
        bool stale = false;
#pragma unroll
        for (int b = 0; b < kRouteRows; ++b) {
          const int e = e0 + b * kConsumerWarps;
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            const int c = 2 * lane + 64 * k;
            if (fepoch(w[b][k][0]) != ep || fepoch(w[b][k][1]) != ep) {
              stale = true;
              const unsigned long long* src = P.froute + (size_t)e * gp + c;
              if (c + 1 < G) ld_flag2(src, w[b][k][0], w[b][k][1]);
              else w[b][k][0] = ld_flag1(src);
            }
          }
        }
        if (!__any_sync(0xffffffffu, stale)) break;
        if (it == 0) {
          t0 = gtimer();
        } else if ((it & 31) == 0) {
          bool give_up = false;
          if (sc->abort || ld_relaxed(&P.ctrl->abort)) {
            give_up = true;
          } else if (gtimer() - t0 > P.timeout_ns) {
            record_error(P, kErrTimeout, 4, step);
            give_up = true;
          }
          if (__any_sync(0xffffffffu, give_up)) {
            sc->abort = 1;
            break;
          }
        }
      }
#pragma unroll
      for (int b = 0; b < kRouteRows; ++b) {
        float a = 0.f;
#pragma unroll
        for (int k = 0; k < 3; ++k) a += fval(w[b][k][0]) + fval(w[b][k][1]);
        a = warp_sum(a);
        const int e = e0 + b * kConsumerWarps;
        if (lane == 0 && e <= E) part[e < E ? e : 2 * kMaxExperts] = a;
      }
    }
    cbar();
    if (warp == 0) {
      // top_k rounds of a warp arg-max over the softmax numerators (the
      // denominator cancels in the renormalisation), larger first and the
      // lower expert index on ties; a chosen expert is struck out with -1
      float* pr = part + kMaxExperts;
      const float inv = 1.0f / sqrtf(part[2 * kMaxExperts] / (float)P.d + P.eps);
      for (int e = lane; e < P.E; e += 32) part[e] *= inv;
      __syncwarp();
      float mx = -INFINITY;
      for (int e = lane; e < P.E; e += 32) mx = fmaxf(mx, part[e]);
      mx = warp_max(mx);
      for (int e = lane; e < P.E; e += 32) pr[e] = expf(part[e] - mx);
      __syncwarp();
      int* re = sc->route_e[route_round % kRouteRing];
      float wsum = 0.f;
      for (int k = 0; k < P.top_k; ++k) {
        float bv = -1.f;
        int bi = INT_MAX;
        for (int e = lane; e < P.E; e += 32)
          if (pr[e] > bv) {
            bv = pr[e];
            bi = e;
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
        if (bi >= P.E) {  // no orderable candidate (a non-finite logit): stop, with a valid index
          bi = k;
          if (lane == 0) record_error(P, kErrDevice, 5, step);
        }
        if (lane == 0) {
          re[k] = bi;
          sc->route_w[k] = bv;
          pr[bi] = -1.f;
        }
        wsum += bv;
        __syncwarp();
      }
      if (lane == 0) {
        for (int k = 0; k < P.top_k; ++k) sc->route_w[k] /= wsum;
        __threadfence_block();
        sc->route_seq = route_round + 1;  // hand the choice to the producer lanes
      }
    }
    cbar();
    ++route_round;
  }

  // The per-token step as a sequence of phases: per layer q/k/v, attention,
  // output projection, FFN up (gate/up or routed experts), FFN down; then the
  // LM head when the step samples. Every phase waits for the flagged input it
  // reads (so it starts as soon as that input's producers are done, with no
  // grid-wide barrier between phases), runs its tiles through the one
  // run_segment call site (one inlined copy of the GEMV code keeps the
  // instruction cache warm), then runs its epilogue, which publishes its
  // output flagged.
  enum PhaseKind { PH_QKV = 0, PH_ATTN = 1, PH_O = 2, PH_UP = 3, PH_DOWN = 4, PH_LM = 5 };

  __device__ void run() {
    const int c = blockIdx.x;
    int tok = P.first_token;
    prefetch_gain(P.attn_norm);
    for (step = 0; step < P.n_steps; ++step) {
      const int pos = P.pos0 + step;
      if (tok < 0 || tok >= P.V) {
        if (tid == 0) record_error(P, kErrDevice, 5, step);
        return;
      }
      const bool lm = step >= P.lm_from_step;
      const __half* erow = P.embed + (size_t)tok * P.d;
      const int nph = P.L * 5 + (lm ? 1 : 0);
      int re[kMaxTopK];
      float rw[kMaxTopK];
      int rpb[kMaxTopK];
      for (int ph = 0; ph < nph; ++ph) {
        const int l = ph / 5;
        const int kind = (l == P.L) ? PH_LM : ph - l * 5;
        tstamp(ph, 0);
        // ---- 1. input vector
        switch (kind) {
          case PH_QKV:
            stage_rope(dc.at(l, 0), pos);
            if (l == 0) load_norm(nullptr, 0u, erow, P.d);
            else load_norm(P.fx + P.d, epoch(l - 1), nullptr, P.d);
            prefetch_gain(P.mlp_norm + (size_t)l * P.d);
            break;
          case PH_O:
            if constexpr (MOE) prefetch_router(l, dc.at(l, 1));
            else prefetch_gate_up(l);
            load_vec(P.fo, epoch(l), P.hq * P.dh);
            break;
          case PH_UP:
            if constexpr (MOE) {
              // routing first: the producer issues the routed experts' tiles
              // while this CTA loads x and runs the shared expert
              const int* pick = sc->route_e[route_round % kRouteRing];
              route(l);
              for (int k = 0; k < P.top_k; ++k) {
                re[k] = pick[k];
                rw[k] = sc->route_w[k];
              }
            }
            load_norm(P.fx, epoch(l), nullptr, P.d);
            if (l + 1 < P.L) prefetch_gain(P.attn_norm + (size_t)(l + 1) * P.d);
            else prefetch_gain(lm ? P.final_norm : P.attn_norm);
            break;
          case PH_DOWN:
            load_vec(P.fh, epoch(l), MOE ? P.ffs + P.top_k * P.ffe : P.ff);
            break;
          case PH_LM:
            load_norm(P.fx + P.d, epoch(P.L - 1), nullptr, P.d);
            prefetch_gain(P.attn_norm);
            break;
          default:
            break;
        }
        if (kind != PH_ATTN) tstamp(ph, 1);  // attention stamps its own input and tile times
        // ---- 2. tiles
        if (kind == PH_ATTN) {
          attention_dispatch(l, pos, ph);
        } else {
          // The LM head and the dense gate/up run in row chunks that fit the
          // partial-sum buffer, each chunk followed by its epilogue (the chunks
          // are whole tile groups: contiguous in the tape and in the
          // producer's tile order). MoE phases run the shared expert and the
          // routed experts as segments. All go through this one run_segment
          // call site.
          const bool chunked = kind == PH_LM || (kind == PH_UP && !MOE);
          const SegDesc& cfull = kind == PH_LM ? dc.at(P.L, 0) : dc.at(l, 2);
          const int csk = kind == PH_LM ? SK_LM : SK_GU;
          const SegShape& csh = P.shp[csk];
          const int crows = chunked ? max(csh.g, (kPartFloats / csh.nk) / csh.g * csh.g) : 1;
          const int nseg = chunked ? (cfull.nrows + crows - 1) / crows
                                   : ((MOE && (kind == PH_UP || kind == PH_DOWN)) ? 1 + P.top_k : 1);
          const float inv = chunked ? norm_scale() : 0.f;
          float v1 = -INFINITY, v2 = -INFINITY;
          int i1 = INT_MAX;
          int pnext = 0;
          for (int si = 0; si < nseg; ++si) {
            SegDesc sub;
            const SegDesc* sd;
            int sk, voff = 0, pbase = 0, pstride, kjbase = 0;
            if (chunked) {
              const int r0 = si * crows;
              sub = SegDesc{cfull.off + (unsigned long long)r0 * csh.K * 2, cfull.row0 + r0,
                            min(crows, cfull.nrows - r0)};
              sd = &sub;
              sk = csk;
            } else if (kind == PH_QKV) { sd = &dc.at(l, 0); sk = SK_QKV; }
            else if (kind == PH_O) { sd = &dc.at(l, 1); sk = SK_O; }
            else if (kind == PH_UP) {
              if (si == 0) { sd = &dc.at(l, 2); sk = SK_SGU; }
              else { sd = &dc.at(l, 4 + re[si - 1]); sk = SK_EGU; pbase = pnext; rpb[si - 1] = pnext; }
            } else {  // PH_DOWN
              if (!MOE) { sd = &dc.at(l, 3); sk = SK_DOWN; }
              else if (si == 0) { sd = &dc.at(l, 3); sk = SK_SDOWN; }
              else {
                sd = &dc.at(l, 4 + P.E + re[si - 1]);
                sk = SK_EDOWN;
                voff = P.ffs + (si - 1) * P.ffe;
                kjbase = P.shp[SK_SDOWN].nk + (si - 1) * P.shp[SK_EDOWN].nk;
              }
            }
            pstride = (kind == PH_DOWN && MOE) ? P.shp[SK_SDOWN].nk + P.top_k * P.shp[SK_EDOWN].nk
                                               : P.shp[sk].nk;
            run_segment(*sd, P.shp[sk], vec + voff / 2, pbase, pstride, kjbase);
            pnext = pbase + sd->nrows * P.shp[sk].nk;
            if (chunked) {
              cbar();
              if (kind == PH_LM) epi_lm_rows(sub, si * crows, inv, v1, i1, v2);
              else epi_swiglu(sub, 0, csh.nk, 0, 1.0f, epoch(l));
              cbar();  // the partial sums are reused by the next chunk
            }
          }
          if (kind == PH_LM) lm_candidates(cfull, v1, i1, v2);
        }
        cbar();
        if (kind != PH_ATTN) tstamp(ph, 2);
        // ---- 3. epilogue
        switch (kind) {
          case PH_QKV:
            epi_qkv(dc.at(l, 0), P.shp[SK_QKV].nk, l, pos);
            break;
          case PH_O:
            epi_residual(dc.at(l, 1), P.shp[SK_O].nk, l == 0 ? erow : nullptr, 0, epoch(l));
            break;
          case PH_UP:
            if constexpr (MOE) {
              epi_swiglu(dc.at(l, 2), 0, P.shp[SK_SGU].nk, 0, 1.0f, epoch(l));
              for (int k = 0; k < P.top_k; ++k)
                epi_swiglu(dc.at(l, 4 + re[k]), rpb[k], P.shp[SK_EGU].nk, P.ffs + k * P.ffe, rw[k], epoch(l));
            }
            break;
          case PH_DOWN:
            epi_residual(dc.at(l, 3), MOE ? P.shp[SK_SDOWN].nk + P.top_k * P.shp[SK_EDOWN].nk : P.shp[SK_DOWN].nk,
                         nullptr, 1, epoch(l));
            break;
          case PH_LM:  // run with the tiles, chunk by chunk
            break;
          default:
            break;
        }
        if (cbar_any(sc->abort != 0)) return;
        tstamp(ph, 3);
      }
      int next;
      if (lm) {
        next = pick_token();
        if (cbar_any(sc->abort != 0)) return;
        if (next == INT_MAX) {  // no finite logit
          if (tid == 0) record_error(P, kErrDevice, 5, step);
          return;
        }
        if (P.forced && P.forced[step] >= 0) next = P.forced[step];
      } else {
        next = P.forced ? P.forced[step] : -1;
      }
      tok = next;
      // one grid barrier per step: it orders this step's KV-cache appends
      // before the next step's bulk copies of them (the phases within a step
      // wait on the flagged words they read instead)
      if (!grid_sync()) return;
    }
    if (c == 0 && tid == 0) P.ctrl->final_token = tok;
  }

  // LM-head epilogue of one row chunk (rows r0 .. of this CTA's LM rows):
  // logits (optional copy out, and kept for sampling) and the thread's
  // running greedy candidate.
  __device__ void epi_lm_rows(const SegDesc& sub, int r0, float inv, float& v1, int& i1, float& v2) {
    const int stride = P.shp[SK_LM].nk;
    const bool sampling = P.samp_temp > 0.f;
    float* keep = sampling ? P.lm_logits + (size_t)blockIdx.x * P.lm_rows + r0 : nullptr;
    for (int r = tid; r < sub.nrows; r += kConsumerThreads) {
      const float y = row_sum(r, stride) * inv;
      const int row = sub.row0 + r;
      if (P.logits_out) P.logits_out[(size_t)step * P.V + row] = y;
      if (sampling) keep[r] = (y == y) ? y : -INFINITY;
      cand_merge(v1, i1, v2, y, row, -INFINITY);
    }
  }

  // This CTA's greedy candidate (value, lowest index, runner-up) published
  // flagged; with sampling also its local top-k.
  __device__ void lm_candidates(const SegDesc& dl, float v1, int i1, float v2) {
    cand_warp_merge(v1, i1, v2);
    if (lane == 0) sc->wcand[warp] = Cand{v1, i1, v2, 0};
    cbar();
    if (tid == 0) {
      float a1 = -INFINITY, a2 = -INFINITY;
      int ai = INT_MAX;
      for (int w = 0; w < kConsumerWarps; ++w)
        cand_merge(a1, ai, a2, sc->wcand[w].v1, sc->wcand[w].i1, sc->wcand[w].v2);
      unsigned long long* cb = P.fcand + (size_t)blockIdx.x * 4;
      st_flag2(cb, a1, __int_as_float(ai), epoch(P.L));
      st_flag2(cb + 2, a2, 0.f, epoch(P.L));
    }
    if (P.samp_temp > 0.f) publish_topk(dl);
  }

  // Sampling, step 1 (every CTA): the CTA's top-k logits by rank (larger
  // value first, then lower index), published as flagged (value, index) word
  // pairs in rank order; ranks past the CTA's rows get (-inf, INT_MAX). The
  // list is padded to an even length, as the reader takes two pairs per load.
  __device__ void publish_topk(const SegDesc& dl) {
    const int K = (P.samp_k + 1) & ~1, n = dl.nrows;
    unsigned long long* dst = P.fsamp + (size_t)blockIdx.x * 2 * kSampleK;
    const unsigned ep = epoch(P.L);
    const float* y_of = P.lm_logits + (size_t)blockIdx.x * P.lm_rows;
    for (int r = tid; r < n; r += kConsumerThreads) {
      const float y = y_of[r];
      int rank = 0;
      for (int q = 0; q < n; ++q) {
        const float z = y_of[q];
        rank += (z > y || (z == y && q < r)) ? 1 : 0;
      }
      if (rank < K) st_flag2(dst + 2 * rank, y, __int_as_float(dl.row0 + r), ep);
    }
    for (int j = n + tid; j < K; j += kConsumerThreads) st_flag2(dst + 2 * j, -INFINITY, __int_as_float(INT_MAX), ep);
  }

  // Sampling, step 2 (CTA 0): merge all CTAs' candidates into the global
  // top-k (radix select of the k-th largest 64-bit order key, 8 bits per
  // pass), sort them, and pick by the definition of the sampling oracle:
  // weights exp(z - max z) with z = logit / temperature, the shortest prefix
  // whose cumulative weight reaches top_p of the total, then the first entry
  // whose cumulative weight exceeds u times the kept total. u comes from
  // Philox4x32-10 with counter (position, 0, 0, 0) and key (seed low, seed
  // high): the top 24 bits of the first word times 2^-24.
  __device__ int sample_select(int pos) {
    constexpr int kSlots = (kSampleMaxGrid * kSampleK + kConsumerThreads - 1) / kConsumerThreads;
    const int K = P.samp_k, n = (int)gridDim.x * K;
    const unsigned ep = epoch(P.L);
    unsigned long long key[kSlots];
#pragma unroll
    for (int sl = 0; sl < kSlots; ++sl) {
      const int c = tid + sl * kConsumerThreads;
      key[sl] = 0ull;
      if (c < n) {
        const int cta = c / K, i = c - cta * K;
        const float4 w = wait4(P.fsamp + (size_t)cta * 2 * kSampleK + 2 * (i & ~1), ep);
        const bool hi = i & 1;
        key[sl] = sample_key(hi ? w.z : w.x, __float_as_int(hi ? w.w : w.y));
      }
    }
    unsigned long long prefix = 0ull, pmask = 0ull;
    int need = K;
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int b = tid; b < 256; b += kConsumerThreads) sc->sel_hist[b] = 0u;
      cbar();
#pragma unroll
      for (int sl = 0; sl < kSlots; ++sl) {
        const int c = tid + sl * kConsumerThreads;
        if (c < n && (key[sl] & pmask) == prefix) atomicAdd(&sc->sel_hist[(key[sl] >> shift) & 255u], 1u);
      }
      cbar();
      if (warp == 0) {
        // lane l scans bins 255 - 8l down to 248 - 8l; bins are taken from the top
        unsigned cnt[8], sum = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          cnt[u] = sc->sel_hist[255 - 8 * lane - u];
          sum += cnt[u];
        }
        unsigned incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const unsigned excl = incl - sum;
        if (excl < (unsigned)need && incl >= (unsigned)need) {
          unsigned acc = excl;
          int bin = 255 - 8 * lane;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (acc + cnt[u] >= (unsigned)need) {
              bin = 255 - 8 * lane - u;
              break;
            }
            acc += cnt[u];
          }
          sc->sel_prefix = prefix | ((unsigned long long)bin << shift);
          sc->sel_need = need - (int)acc;
        }
      }
      cbar();
      prefix = sc->sel_prefix;
      need = sc->sel_need;
      pmask |= 0xFFull << shift;
    }
    // prefix is now the k-th largest key: gather the K keys >= it and sort them
    if (tid == 0) sc->sel_count = 0;
    cbar();
#pragma unroll
    for (int sl = 0; sl < kSlots; ++sl) {
      const int c = tid + sl * kConsumerThreads;
      if (c < n && key[sl] >= prefix) {
        const int at = atomicAdd(&sc->sel_count, 1);
        if (at < kSampleK) sc->sel_key[at] = key[sl];
      }
    }
    cbar();
    unsigned long long mine = 0ull;
    int rank = 0;
    if (tid < K) {
      mine = sc->sel_key[tid];
      for (int q = 0; q < K; ++q) rank += sc->sel_key[q] > mine ? 1 : 0;
    }
    cbar();
    if (tid < K) sc->sel_key[rank] = mine;
    cbar();
    if (warp == 0) {
      const float invT = 1.0f / P.samp_temp;
      const unsigned long long ka = lane < K ? sc->sel_key[lane] : 0ull;
      const unsigned long long kb = lane + 32 < K ? sc->sel_key[lane + 32] : 0ull;
      const float zmax = __shfl_sync(0xffffffffu, key_value(ka), 0) * invT;
      const float wa = lane < K ? expf(key_value(ka) * invT - zmax) : 0.f;
      const float wb = lane + 32 < K ? expf(key_value(kb) * invT - zmax) : 0.f;
      float ca = wa, cb = wb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float ta = __shfl_up_sync(0xffffffffu, ca, o), tb = __shfl_up_sync(0xffffffffu, cb, o);
        if (lane >= o) {
          ca += ta;
          cb += tb;
        }
      }
      const float totA = __shfl_sync(0xffffffffu, ca, 31);
      cb += totA;  // entries lane + 32 follow all of the first 32
      const float tot = __shfl_sync(0xffffffffu, cb, 31);
      // cut: the last kept entry
      int cut = K - 1;
      if (P.samp_p < 1.f) {
        const float lim = P.samp_p * tot;
        const unsigned ma = __ballot_sync(0xffffffffu, lane < K && ca >= lim);
        const unsigned mb = __ballot_sync(0xffffffffu, lane + 32 < K && cb >= lim);
        cut = ma ? __ffs(ma) - 1 : (mb ? 32 + __ffs(mb) - 1 : K - 1);
      }
      const float kept = cut < 32 ? __shfl_sync(0xffffffffu, ca, cut) : __shfl_sync(0xffffffffu, cb, cut - 32);
      const uint32_t w0 = philox_w0((uint32_t)pos, 0u, 0u, 0u, (uint32_t)P.samp_seed, (uint32_t)(P.samp_seed >> 32));
      const float target = (float)(w0 >> 8) * (1.0f / 16777216.0f) * kept;
      const unsigned pa = __ballot_sync(0xffffffffu, lane <= cut && lane < K && ca > target);
      const unsigned pb = __ballot_sync(0xffffffffu, lane + 32 <= cut && lane + 32 < K && cb > target);
      const int pick = pa ? __ffs(pa) - 1 : (pb ? 32 + __ffs(pb) - 1 : cut);
      const unsigned long long kp = pick < 32 ? __shfl_sync(0xffffffffu, ka, pick) : __shfl_sync(0xffffffffu, kb, pick - 32);
      if (lane == 0) sc->sel_count = key_index(kp);
    }
    cbar();
    return sc->sel_count;
  }

  // Every CTA reduces all CTAs' flagged candidates the same way.
  __device__ int pick_token() {
    float v1 = -INFINITY, v2 = -INFINITY;
    int i1 = INT_MAX;
    for (int cc = tid; cc < (int)gridDim.x; cc += kConsumerThreads) {
      const float4 cv = wait4(P.fcand + (size_t)cc * 4, epoch(P.L));
      cand_merge(v1, i1, v2, cv.x, __float_as_int(cv.y), cv.z);
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
      if (blockIdx.x == 0) {
        if (P.samp_temp <= 0.f) P.out_tokens[step] = ai;
        if (P.margins_out) P.margins_out[step] = a1 - a2;
      }
    }
    cbar();
    if (P.samp_temp > 0.f && sc->tok != INT_MAX) {
      // CTA 0 samples and publishes the token; the others wait for its word
      unsigned long long* tw = P.fsamp + (size_t)gridDim.x * 2 * kSampleK;
      if (blockIdx.x == 0) {
        const int t = sample_select(P.pos0 + step);
        if (tid == 0) {
          P.out_tokens[step] = t;
          st_flag2(tw, __int_as_float(t), 0.f, epoch(P.L));
          st_flag2(tw + 2, 0.f, 0.f, epoch(P.L));
          sc->tok = t;
        }
      } else if (tid == 0) {
        sc->tok = __float_as_int(wait4(tw, epoch(P.L)).x);
      }
      cbar();
    }
    return sc->tok;
  }
};

template <int HD, bool MOE>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) unsigned char smem[];
  SmemCtl* sc = reinterpret_cast<SmemCtl*>(smem);
  float* part = reinterpret_cast<float*>(smem + smem_ctl_bytes());
  float* vec = part + kPartFloats;
  SegDesc* dsm = reinterpret_cast<SegDesc*>(smem + smem_desc_offset(P.vec_floats));
  unsigned char* ring = smem + smem_ring_offset(P.vec_floats, 4 * P.L + 1);
  const SegDesc* dg = P.desc + (size_t)blockIdx.x * (P.L * P.slots + 1);
  for (int i = threadIdx.x; i <= 4 * P.L; i += kThreads)
    dsm[i] = (i < 4 * P.L) ? dg[(size_t)(i >> 2) * P.slots + (i & 3)] : dg[(size_t)P.L * P.slots];
  const DescCache dc{dsm, dg, P.L, P.slots};
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.n_stages; ++s) {
      mbar_init(&sc->full[s], 1);
      mbar_init(&sc->empty[s], 1);
    }
    sc->route_seq = 0;
    sc->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x >= kConsumerThreads) {
    const int lane = threadIdx.x - kConsumerThreads;
    if (lane < P.n_stages) {
      Producer<MOE> pr(P, sc, ring, lane, dc);
      pr.run();
    }
  } else {
    Consumer<HD, MOE> cs(P, sc, part, vec, ring, dc);
    cs.run();
  }
}

}  // namespace kie
