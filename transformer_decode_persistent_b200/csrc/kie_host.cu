// Host side of libkie: context, weight packer, launcher and the C ABI.
//
// The packer lays every matrix out as the per-CTA "weight tape" that the
// persistent kernel streams with TMA bulk copies (tile format in
// kie_internal.h); the launcher runs a whole prefill or n-token decode as ONE
// cooperative launch, so the host is crossed once per call instead of once per
// kernel (the pages put a kernel launch at ~4.5 us and count >1,100 us of
// launch overhead per token for an unfused 25-layer stack: "メモリの壁を打破する：
// 標準的なGPUで3,000 tokens/sの推論を実現する", section "マイクロ秒が失われる場所").
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/kie.h"
#include "kie_internal.h"
#include "prefill.h"

namespace kie {
int kernel_smem_bytes(int vec_floats, int n_desc, int n_stages, int stage_bytes);
int kernel_max_stages();
const void* kernel_entry_128_0();
const void* kernel_entry_128_1();
const void* kernel_entry_64_0();
const void* kernel_entry_64_1();
// the decode kernel compiled for this head_dim and FFN kind (decode_inst.cu)
inline const void* kernel_entry(int head_dim, bool moe) {
  if (head_dim == 128) return moe ? kernel_entry_128_1() : kernel_entry_128_0();
  return moe ? kernel_entry_64_1() : kernel_entry_64_0();
}
}  // namespace kie

using namespace kie;

namespace {

thread_local std::string g_create_error;

}  // namespace

struct kie_ctx {
  kie_config cfg{};
  int device = 0;
  int sms = 0;
  int grid = 0;
  int n_stages = 0;
  int stage_bytes = 0;
  int xplane = 0;          // float offset of the input vector's second plane
  int vec_floats = 0;
  int gbuf_off = 0;
  int rslice_off = 0;      // MoE router slice (floats into the vector buffer)
  int rslice_rows = 0;
  int smem = 0;
  int max_chunks = 0;
  int hbuf = 0;
  int slots = 0;
  SegShape shp[SK_COUNT]{};
  // device memory
  std::vector<void*> allocs;
  unsigned char* tape = nullptr;
  size_t tape_bytes = 0;
  SegDesc* desc = nullptr;
  __half *embed = nullptr, *attn_norm = nullptr, *mlp_norm = nullptr, *final_norm = nullptr,
         *router = nullptr;
  __half *kcache = nullptr, *vcache = nullptr;
  float2* rope = nullptr;
  unsigned long long* fsamp = nullptr;  // sampling candidates (allocated on first use)
  size_t fsamp_bytes = 0;
  float* lm_logits = nullptr;           // sampling: per-CTA LM-head logits of a step
  int lm_rows = 0;                      // most LM-head rows of one CTA
  // Ctrl | flagged scratch (fx, fq, fo, fh, fcand, attention chunk records), cleared before every launch
  unsigned char* syncblk = nullptr;
  size_t syncblk_bytes = 0;
  int *tok_dev = nullptr, *forced_dev = nullptr;
  float* margins_dev = nullptr;
  // state
  bool loaded = false;
  bool poisoned = false;
  int32_t pos = 0;
  int32_t pending = -1;
  int64_t launches = 0;
  int64_t stream_bytes = 0;
  std::string err;
  // tensor-core prompt prefill: row-major layer matrices in the packed row
  // orders (q/k/v RoPE pairs and gate/up pairs adjacent), activation buffers
  // for one chunk, and their tensor maps
  bool pf_ready = false;
  // [L][rows][K]: q/k/v, o, gate/up, down (MoE: the shared expert's gate/up and down)
  __half *pf_w[4] = {nullptr, nullptr, nullptr, nullptr};
  // MoE: the routed experts' [L][E][rows][K] gate/up and down, the router
  // [L][E rounded up to a GEMM tile][d] (zero rows past E), routing buffers,
  // the expert-sorted activations and hidden rows, the experts' outputs
  __half *pf_we[2] = {nullptr, nullptr};
  __half* pf_router = nullptr;
  int pf_epad = 0;
  float *pf_logits = nullptr, *pf_wt = nullptr, *pf_y = nullptr;
  int *pf_sel = nullptr, *pf_range = nullptr, *pf_rowof = nullptr, *pf_tokof = nullptr;
  __half *pf_gh = nullptr, *pf_gl = nullptr, *pf_eh = nullptr, *pf_el = nullptr;
  std::vector<CUtensorMap> pf_emap;  // [L][E][2]
  std::vector<CUtensorMap> pf_rmap;  // [L]
  CUtensorMap pf_map_gh{}, pf_map_gl{}, pf_map_eh{}, pf_map_el{};
  float *pf_x = nullptr, *pf_q = nullptr;
  __half *pf_xh = nullptr, *pf_xl = nullptr, *pf_oh = nullptr, *pf_ol = nullptr, *pf_hh = nullptr, *pf_hl = nullptr;
  int *pf_tok = nullptr, *pf_err = nullptr;
  std::vector<CUtensorMap> pf_wmap;  // [L][4]
  CUtensorMap pf_map_xh{}, pf_map_xl{}, pf_map_oh{}, pf_map_ol{}, pf_map_hh{}, pf_map_hl{};
};

namespace {

kie_status fail(kie_ctx* c, kie_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (c) c->err = buf;
  else g_create_error = buf;
  return s;
}

#define CUDA_TRY(ctx, call)                                                                  \
  do {                                                                                       \
    cudaError_t e_ = (call);                                                                 \
    if (e_ != cudaSuccess) {                                                                 \
      return fail((ctx), e_ == cudaErrorMemoryAllocation ? KIE_ERR_OOM : KIE_ERR_CUDA,      \
                  "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__); \
    }                                                                                        \
  } while (0)

template <class T>
kie_status dalloc(kie_ctx* c, T** p, size_t bytes) {
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, bytes ? bytes : 16);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(c, e == cudaErrorMemoryAllocation ? KIE_ERR_OOM : KIE_ERR_CUDA,
                "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
  }
  c->allocs.push_back(q);
  *p = static_cast<T*>(q);
  return KIE_OK;
}

void dfree(kie_ctx* c, void* p) {
  if (!p) return;
  auto it = std::find(c->allocs.begin(), c->allocs.end(), p);
  if (it != c->allocs.end()) c->allocs.erase(it);
  cudaFree(p);
}

// CUDA device owning `p` (device or managed memory), or -1 for host memory.
int ptr_device(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) ? a.device : -1;
}

bool is_device_ptr(const void* p) { return ptr_device(p) >= 0; }

// INVALID_ARG if `p` is device memory of a device other than the context's.
kie_status check_own_device(kie_ctx* c, const void* p, const char* what) {
  const int dev = p ? ptr_device(p) : -1;
  if (dev >= 0 && dev != c->device)
    return fail(c, KIE_ERR_INVALID_ARG, "%s is memory of device %d; the context is on device %d", what, dev,
                c->device);
  return KIE_OK;
}

// Tile shape for a segment kind: rows per tile g and column chunks nk. Prefer
// g >= 4 (the input vector chunk is reused across g rows) with the fewest
// chunks; GU kinds need an even g so (gate, up) pairs share a tile.
SegShape choose_shape(int K, bool pairs, int stage_bytes) {
  // Preferred: column blocks of 512 halves (two 16-byte chunks per lane, up to
  // kMaxRowsWide rows) or of 768 halves (three chunks, up to 8 rows): the
  // kernel's register-blocked tile GEMVs for these widths take any row count.
  if (K % 512 == 0 && stage_bytes / 1024 >= 4)
    return SegShape{K, std::min(kMaxRowsWide, stage_bytes / 1024), K / 512, 512};
  if (K % 768 == 0 && stage_bytes / 1536 >= 4)
    return SegShape{K, std::min(kMaxRowsPerTile, stage_bytes / 1536), K / 768, 768};
  // First choice: the fewest column blocks that give at least 4 rows per
  // tile. A split into more blocks wins when its chunks divide evenly over the
  // 32 lanes (kc a multiple of 256 halves, so the kernel's copy-out GEMV
  // applies) and its tiles keep at least 3/4 of the first choice's bytes.
  // With no 4-row split, the tallest tile.
  auto at = [&](int nk) {
    SegShape sh{K, 0, nk, 0};
    if (K % nk || (K / nk) % 8) return sh;
    sh.kc = K / nk;
    int g = std::min(kMaxRowsPerTile, stage_bytes / (2 * sh.kc));
    if (pairs) g &= ~1;
    sh.g = std::max(g, 0);
    return sh;
  };
  SegShape best{K, 0, 0, 0}, first4{K, 0, 0, 0};
  for (int nk = 1; nk <= 64; ++nk) {
    const SegShape sh = at(nk);
    if (sh.g < 1) continue;
    if (sh.g >= 4 && first4.g == 0) first4 = sh;
    if (sh.g > best.g) best = sh;
  }
  if (!first4.g) return best;
  if (first4.kc % 256 == 0) return first4;
  for (int nk = first4.nk + 1; nk <= 64; ++nk) {
    const SegShape sh = at(nk);
    if (sh.g >= 4 && sh.kc % 256 == 0 && 4LL * sh.g * sh.kc >= 3LL * first4.g * first4.kc) return sh;
  }
  return first4;
}

// Tile height evened out over the rows one CTA holds (`rows` split over
// `grid` CTAs in units of 1 or 2 rows): as few tiles as the chosen height
// allows, all about the same height, so no tile is a sliver.
SegShape balance_rows(SegShape sh, int rows, int per, bool pairs, int grid) {
  const int maxu = (rows / per + grid - 1) / grid;
  const int maxrows = std::max(1, maxu * per);
  const int ngroups = (maxrows + sh.g - 1) / sh.g;
  int g = (maxrows + ngroups - 1) / ngroups;
  if (pairs) g = (g + 1) & ~1;
  if (g >= 1 && g <= sh.g) sh.g = g;
  return sh;
}

// Rows are handed to CTAs in units: (gate, up) pairs for the FFN kinds and
// RoPE pairs (dims i, i + dh/2 of one head) for q/k/v.
int seg_rows_per_unit(int kind) {
  return (kind == SK_GU || kind == SK_SGU || kind == SK_EGU || kind == SK_QKV) ? 2 : 1;
}

struct Tensor {
  const void* data;
  int64_t rows, cols;
  bool on_dev;
};

}  // namespace

// ------------------------------------------------------------------- packing

__global__ void pack_rows_kernel(const unsigned long long* __restrict__ src,
                                 const unsigned long long* __restrict__ dst, const int* __restrict__ n16,
                                 long long count) {
  const int lane = threadIdx.x & 31;
  long long w = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const long long stride = (long long)gridDim.x * (blockDim.x / 32);
  for (; w < count; w += stride) {
    const uint4* s = reinterpret_cast<const uint4*>(src[w]);
    uint4* d = reinterpret_cast<uint4*>(dst[w]);
    const int n = n16[w];
    for (int i = lane; i < n; i += 32) d[i] = s[i];
  }
}

namespace {

struct Planner {
  const kie_config& k;
  int G;
  int slots;
  std::vector<SegDesc> desc;  // [G][L*slots + 1]

  Planner(const kie_config& cfg, int grid, int nslots) : k(cfg), G(grid), slots(nslots) {
    desc.assign((size_t)G * (k.n_layers * slots + 1), SegDesc{0, 0, 0});
  }

  // rows of kind over the (virtual) row space, split into G near-equal ranges;
  // the CTAs that get one extra unit rotate with `rot` so no CTA is always heavy.
  void assign(int l, int slot, int kind, int rows, int rot) {
    const int per = seg_rows_per_unit(kind);
    const int U = rows / per;
    const int b = U / G, rem = U % G;
    for (int ci = 0; ci < G; ++ci) {
      const int rank = (ci + rot) % G;
      const int u0 = rank * b + std::min(rank, rem);
      const int nu = b + (rank < rem ? 1 : 0);
      SegDesc& d = desc[(size_t)ci * (k.n_layers * slots + 1) + (size_t)l * slots + slot];
      d.row0 = u0 * per;
      d.nrows = nu * per;
    }
    (void)kind;
  }
};

// Segment kind of descriptor slot `slot` of layer l (l == L: the LM head).
int kind_of(const kie_config& k, int l, int slot) {
  if (l == k.n_layers) return SK_LM;
  if (slot == 0) return SK_QKV;
  if (slot == 1) return SK_O;
  if (k.n_experts == 0) return slot == 2 ? SK_GU : SK_DOWN;
  if (slot == 2) return SK_SGU;
  if (slot == 3) return SK_SDOWN;
  return slot < 4 + k.n_experts ? SK_EGU : SK_EDOWN;
}

// The weight-tape plan for `grid` CTAs with ring stages of `sb` bytes: the
// tile shape of every segment kind, each CTA's row range of every matrix
// (desc, [grid][L*slots + 1]) and its byte offset in the tape (each CTA's
// region contiguous, segments in execution order). Pure host arithmetic.
struct Plan {
  SegShape shp[SK_COUNT] = {};
  std::vector<SegDesc> desc;
  size_t tape_bytes = 0;
  int slots = 0;
};

kie_status make_plan(kie_ctx* c, const kie_config& k, int G, int sb, Plan& plan) {
  const bool moe = k.n_experts > 0;
  const int d = k.d_model, hq = k.n_heads, hk = k.n_kv_heads, dh = k.head_dim, L = k.n_layers;
  const int ffs = k.ffn_shared, ffe = k.ffn_expert;
  SegShape* shp = plan.shp;
  shp[SK_QKV] = balance_rows(choose_shape(d, false, sb), (hq + 2 * hk) * dh, 2, false, G);
  shp[SK_O] = balance_rows(choose_shape(hq * dh, false, sb), d, 1, false, G);
  shp[SK_LM] = balance_rows(choose_shape(d, false, sb), k.vocab, 1, false, G);
  if (!moe) {
    shp[SK_GU] = balance_rows(choose_shape(d, true, sb), 2 * k.ffn, 2, true, G);
    shp[SK_DOWN] = balance_rows(choose_shape(k.ffn, false, sb), d, 1, false, G);
  } else {
    shp[SK_SGU] = balance_rows(choose_shape(d, true, sb), 2 * ffs, 2, true, G);
    shp[SK_EGU] = balance_rows(choose_shape(d, true, sb), 2 * ffe, 2, true, G);
    shp[SK_SDOWN] = balance_rows(choose_shape(ffs, false, sb), d, 1, false, G);
    shp[SK_EDOWN] = balance_rows(choose_shape(ffe, false, sb), d, 1, false, G);
  }
  for (int i = 0; i < SK_COUNT; ++i)
    if (shp[i].K && shp[i].g < 1)
      return fail(c, KIE_ERR_INVALID_ARG, "no tile shape of %d columns fits a %d-byte ring stage", shp[i].K, sb);

  // row assignment
  plan.slots = slots_per_layer(moe ? k.n_experts : 0);
  Planner pl(k, G, plan.slots);
  for (int l = 0; l < L; ++l) {
    const int rot = (int)(((long long)l * 53) % G);
    pl.assign(l, 0, SK_QKV, (hq + 2 * hk) * dh, rot);
    // the output and down projections own the same residual rows in every
    // layer (no rotation): each CTA keeps its rows in shared memory
    pl.assign(l, 1, SK_O, d, 0);
    if (!moe) {
      pl.assign(l, 2, SK_GU, 2 * k.ffn, (rot + 31) % G);
      pl.assign(l, 3, SK_DOWN, d, 0);
    } else {
      pl.assign(l, 2, SK_SGU, 2 * ffs, (rot + 31) % G);
      pl.assign(l, 3, SK_SDOWN, d, 0);
      for (int e = 0; e < k.n_experts; ++e) {
        pl.assign(l, 4 + e, SK_EGU, 2 * ffe, (rot + 97 + 7 * e) % G);
        pl.assign(l, 4 + k.n_experts + e, SK_EDOWN, d, 0);
      }
    }
  }
  pl.assign(L, 0, SK_LM, k.vocab, 0);

  const int slots = plan.slots;
  const int per_cta = L * slots + 1;
  // partial-slot capacity per phase
  {
    int worst = 0;
    for (int ci = 0; ci < G; ++ci) {
      const SegDesc* D = &pl.desc[(size_t)ci * per_cta];
      for (int l = 0; l < L; ++l) {
        const SegDesc* Dl = D + (size_t)l * slots;
        worst = std::max(worst, Dl[0].nrows * shp[SK_QKV].nk);
        worst = std::max(worst, Dl[1].nrows * shp[SK_O].nk);
        if (!moe) {
          // gate/up runs in row chunks: one tile group of partial sums must fit
          worst = std::max(worst, std::min(Dl[2].nrows, shp[SK_GU].g) * shp[SK_GU].nk);
          worst = std::max(worst, Dl[3].nrows * shp[SK_DOWN].nk);
        } else {
          int eg = 0;
          for (int e = 0; e < k.n_experts; ++e) eg = std::max(eg, Dl[4 + e].nrows);
          worst = std::max(worst, Dl[2].nrows * shp[SK_SGU].nk + k.top_k * eg * shp[SK_EGU].nk);
          worst = std::max(worst, Dl[3].nrows * (shp[SK_SDOWN].nk + k.top_k * shp[SK_EDOWN].nk));
        }
      }
      // the LM head runs in row chunks too
      worst = std::max(worst, std::min(D[(size_t)L * slots].nrows, shp[SK_LM].g) * shp[SK_LM].nk);
    }
    if (worst > kPartFloats)
      return fail(c, KIE_ERR_INVALID_ARG, "a CTA would hold %d partial sums (max %d)", worst, kPartFloats);
  }

  // tape offsets: each CTA's region contiguous, segments in execution order
  size_t off = 0;
  for (int ci = 0; ci < G; ++ci) {
    for (int l = 0; l <= L; ++l) {
      const int ns = (l == L) ? 1 : slots;
      for (int slot = 0; slot < ns; ++slot) {
        SegDesc& sd = pl.desc[(size_t)ci * per_cta + (size_t)l * slots + slot];
        sd.off = off;
        off += (size_t)sd.nrows * shp[kind_of(k, l, slot)].K * 2;
      }
    }
  }
  plan.tape_bytes = off;
  plan.desc = std::move(pl.desc);
  return KIE_OK;
}

// The region cleared before every launch: control block and the flagged
// scratch words (see Params).
struct SyncLayout {
  size_t fx, fq, fo, fh, fcand, apart, froute, total;
};

SyncLayout sync_layout(const kie_config& k, int grid, int hbuf, int max_chunks) {
  auto a16 = [](size_t b) { return (b + 15) & ~(size_t)15; };
  SyncLayout L{};
  size_t off = a16(sizeof(Ctrl));
  L.fx = off;    off += (size_t)2 * k.d_model * 8;
  L.fq = off;    off += (size_t)(k.n_heads + 2 * k.n_kv_heads) * k.head_dim * 8;
  L.fo = off;    off += (size_t)k.n_heads * k.head_dim * 8;
  L.fh = off;    off += (size_t)hbuf * 8;
  L.fcand = off; off += (size_t)grid * 4 * 8;
  L.apart = off; off += (size_t)k.n_heads * max_chunks * (k.head_dim + 4) * 8;
  L.froute = off; off += k.n_experts ? (size_t)(k.n_experts + 1) * ((grid + 1) & ~1) * 8 : 0;
  L.total = off;
  return L;
}

void set_sync_params(Params& P, unsigned char* base, const SyncLayout& L) {
  P.ctrl = reinterpret_cast<Ctrl*>(base);
  P.apart = reinterpret_cast<unsigned long long*>(base + L.apart);
  P.fx = reinterpret_cast<unsigned long long*>(base + L.fx);
  P.fq = reinterpret_cast<unsigned long long*>(base + L.fq);
  P.fo = reinterpret_cast<unsigned long long*>(base + L.fo);
  P.fh = reinterpret_cast<unsigned long long*>(base + L.fh);
  P.fcand = reinterpret_cast<unsigned long long*>(base + L.fcand);
  P.froute = reinterpret_cast<unsigned long long*>(base + L.froute);
}

// Shape checks shared by kie_create and kie_plan (messages via kie_last_error(NULL)).
kie_status validate_config(const kie_config& k) {
  const bool moe = k.n_experts > 0;
  if (k.n_layers < 1 || k.d_model < 8 || k.n_heads < 1 || k.n_kv_heads < 1 || k.head_dim < 2 ||
      k.vocab < 2 || k.max_ctx < 1)
    return fail(nullptr, KIE_ERR_INVALID_ARG, "non-positive model dimension");
  if (k.d_model % 8 || (k.n_heads * k.head_dim) % 8)
    return fail(nullptr, KIE_ERR_INVALID_ARG, "d_model and n_heads*head_dim must be multiples of 8");
  if (!(k.head_dim == 64 || k.head_dim == 128))
    return fail(nullptr, KIE_ERR_INVALID_ARG, "head_dim must be 64 or 128");
  if (k.n_kv_heads > k.n_heads)
    return fail(nullptr, KIE_ERR_INVALID_ARG, "n_kv_heads > n_heads");
  // a KV head's query heads are attended in sub-units of at most
  // kMaxHeadsPerGroup (the kernel's attention plan); every sub-unit needs one
  {
    const int gmax = (k.n_heads + k.n_kv_heads - 1) / k.n_kv_heads;
    const int sub = (gmax + kMaxHeadsPerGroup - 1) / kMaxHeadsPerGroup, hs = (gmax + sub - 1) / sub;
    for (int g = 0; g < k.n_kv_heads; ++g) {
      const int lo = (g * k.n_heads + k.n_kv_heads - 1) / k.n_kv_heads;
      const int hi = ((g + 1) * k.n_heads + k.n_kv_heads - 1) / k.n_kv_heads;
      if (hi - lo < 1 || (sub - 1) * hs >= hi - lo || gmax > kMaxQueryHeadsPerKv)
        return fail(nullptr, KIE_ERR_INVALID_ARG,
                    "KV head %d serves %d query heads (1..%d allowed, in sub-units of at most %d)", g, hi - lo,
                    kMaxQueryHeadsPerKv, kMaxHeadsPerGroup);
    }
  }
  if (moe) {
    if (k.ffn != 0 || k.top_k < 1 || k.top_k > kMaxTopK || k.top_k > k.n_experts ||
        k.n_experts > kMaxExperts || k.ffn_expert < 8 || k.ffn_expert % 8 || k.ffn_shared < 0 ||
        k.ffn_shared % 8)
      return fail(nullptr, KIE_ERR_INVALID_ARG, "bad MoE shape");
  } else {
    if (k.ffn < 8 || k.ffn % 8 || k.top_k || k.ffn_expert || k.ffn_shared)
      return fail(nullptr, KIE_ERR_INVALID_ARG, "bad dense FFN shape");
  }
  if (!(k.rms_eps >= 0.f) || !(k.rope_theta > 0.f))
    return fail(nullptr, KIE_ERR_INVALID_ARG, "bad rms_eps / rope_theta");

  return KIE_OK;
}

}  // namespace

// Buffers and tensor maps of the tensor-core prefill, once the prefill weights
// exist. `ff` is the dense FFN width, or the MoE shared expert's (0: none).
static kie_status prefill_setup(kie_ctx* c) {
  using namespace kie::pf;
  const kie_config& k = c->cfg;
  const bool moe = k.n_experts > 0;
  const int d = k.d_model, hq = k.n_heads, hk = k.n_kv_heads, dh = k.head_dim, L = k.n_layers;
  const int ff = moe ? k.ffn_shared : k.ffn, E = k.n_experts, ffe = k.ffn_expert, rows = kChunk * k.top_k;
  kie_status s;
  if (moe && !c->pf_logits) {
    if ((s = dalloc(c, &c->pf_logits, (size_t)kChunk * E * 4)) || (s = dalloc(c, &c->pf_wt, (size_t)rows * 4)) ||
        (s = dalloc(c, &c->pf_y, (size_t)rows * d * 4)) || (s = dalloc(c, &c->pf_sel, (size_t)rows * 4)) ||
        (s = dalloc(c, &c->pf_range, (size_t)E * 2 * 4)) || (s = dalloc(c, &c->pf_rowof, (size_t)rows * 4)) ||
        (s = dalloc(c, &c->pf_tokof, (size_t)rows * 4)) || (s = dalloc(c, &c->pf_gh, (size_t)rows * d * 2)) ||
        (s = dalloc(c, &c->pf_gl, (size_t)rows * d * 2)) || (s = dalloc(c, &c->pf_eh, (size_t)rows * ffe * 2)) ||
        (s = dalloc(c, &c->pf_el, (size_t)rows * ffe * 2)))
      return s;
    // rows past an expert's range are read by its last GEMM tile (their
    // columns are discarded); keep them finite
    CUDA_TRY(c, cudaMemset(c->pf_gh, 0, (size_t)rows * d * 2));
    CUDA_TRY(c, cudaMemset(c->pf_gl, 0, (size_t)rows * d * 2));
    CUDA_TRY(c, cudaMemset(c->pf_eh, 0, (size_t)rows * ffe * 2));
    CUDA_TRY(c, cudaMemset(c->pf_el, 0, (size_t)rows * ffe * 2));
  }
  if (!c->pf_x) {
    if ((s = dalloc(c, &c->pf_x, (size_t)kChunk * d * 4)) || (s = dalloc(c, &c->pf_q, (size_t)kChunk * hq * dh * 4)) ||
        (s = dalloc(c, &c->pf_xh, (size_t)kChunk * d * 2)) || (s = dalloc(c, &c->pf_xl, (size_t)kChunk * d * 2)) ||
        (s = dalloc(c, &c->pf_oh, (size_t)kChunk * hq * dh * 2)) ||
        (s = dalloc(c, &c->pf_ol, (size_t)kChunk * hq * dh * 2)) ||
        (ff && (s = dalloc(c, &c->pf_hh, (size_t)kChunk * ff * 2))) ||
        (ff && (s = dalloc(c, &c->pf_hl, (size_t)kChunk * ff * 2))) ||
        (s = dalloc(c, &c->pf_tok, (size_t)kChunk * 4)) || (s = dalloc(c, &c->pf_err, 16)))
      return s;
    // rows past a chunk's length are read by the last GEMM tile (their
    // columns are discarded); keep them finite
    CUDA_TRY(c, cudaMemset(c->pf_xh, 0, (size_t)kChunk * d * 2));
    CUDA_TRY(c, cudaMemset(c->pf_xl, 0, (size_t)kChunk * d * 2));
    CUDA_TRY(c, cudaMemset(c->pf_oh, 0, (size_t)kChunk * hq * dh * 2));
    CUDA_TRY(c, cudaMemset(c->pf_ol, 0, (size_t)kChunk * hq * dh * 2));
    if (ff) {
      CUDA_TRY(c, cudaMemset(c->pf_hh, 0, (size_t)kChunk * ff * 2));
      CUDA_TRY(c, cudaMemset(c->pf_hl, 0, (size_t)kChunk * ff * 2));
    }
    CUDA_TRY(c, cudaMemset(c->pf_err, 0, 16));
  }
  bool ok = make_map(&c->pf_map_xh, c->pf_xh, kChunk, d, kBN) && make_map(&c->pf_map_xl, c->pf_xl, kChunk, d, kBN) &&
            make_map(&c->pf_map_oh, c->pf_oh, kChunk, hq * dh, kBN) &&
            make_map(&c->pf_map_ol, c->pf_ol, kChunk, hq * dh, kBN) &&
            (!ff || (make_map(&c->pf_map_hh, c->pf_hh, kChunk, ff, kBN) &&
                     make_map(&c->pf_map_hl, c->pf_hl, kChunk, ff, kBN)));
  const int prow[4] = {(hq + 2 * hk) * dh, d, 2 * ff, d};
  const int pk[4] = {d, hq * dh, d, ff};
  c->pf_wmap.assign((size_t)L * 4, CUtensorMap{});
  for (int l = 0; l < L && ok; ++l)
    for (int m = 0; m < 4 && ok; ++m)
      if (m < 2 || ff)
        ok = make_map(&c->pf_wmap[(size_t)l * 4 + m], c->pf_w[m] + (size_t)l * prow[m] * pk[m], prow[m], pk[m], kBM);
  if (moe && ok) {
    ok = make_map(&c->pf_map_gh, c->pf_gh, rows, d, kBN) && make_map(&c->pf_map_gl, c->pf_gl, rows, d, kBN) &&
         make_map(&c->pf_map_eh, c->pf_eh, rows, ffe, kBN) && make_map(&c->pf_map_el, c->pf_el, rows, ffe, kBN);
    c->pf_emap.assign((size_t)L * E * 2, CUtensorMap{});
    c->pf_rmap.assign((size_t)L, CUtensorMap{});
    for (int l = 0; l < L && ok; ++l) {
      ok = make_map(&c->pf_rmap[l], c->pf_router + (size_t)l * c->pf_epad * d, c->pf_epad, d, kBM);
      for (int e = 0; e < E && ok; ++e) {
        const size_t ge = (size_t)l * E + e;
        ok = make_map(&c->pf_emap[ge * 2], c->pf_we[0] + ge * 2 * ffe * d, 2 * ffe, d, kBM) &&
             make_map(&c->pf_emap[ge * 2 + 1], c->pf_we[1] + ge * d * ffe, d, ffe, kBM);
      }
    }
  }
  if (!ok) return fail(c, KIE_ERR_CUDA, "tensor map encoding for the prefill failed");
  c->pf_ready = true;
  return KIE_OK;
}

// Forward the committed prompt tokens `seq` at positions pos .. pos + n - 1
// through the tensor-core path, filling the KV cache (one chunk of up to
// kChunk tokens at a time; each chunk attends to the cache of the earlier ones).
static kie_status prefill_tc(kie_ctx* c, const std::vector<int32_t>& seq, cudaStream_t st) {
  using namespace kie::pf;
  const kie_config& k = c->cfg;
  const bool moe = k.n_experts > 0;
  const int d = k.d_model, hq = k.n_heads, hk = k.n_kv_heads, dh = k.head_dim, L = k.n_layers;
  const int ff = moe ? k.ffn_shared : k.ffn, E = k.n_experts, ffe = k.ffn_expert, K = k.top_k;
  const int qkv_rows = (hq + 2 * hk) * dh;
  CUDA_TRY(c, cudaMemsetAsync(c->pf_err, 0, 4, st));
  for (size_t c0 = 0; c0 < seq.size(); c0 += kChunk) {
    const int T = (int)std::min<size_t>(kChunk, seq.size() - c0);
    const int p0 = c->pos + (int)c0;
    CUDA_TRY(c, cudaMemcpyAsync(c->pf_tok, seq.data() + c0, (size_t)T * 4, cudaMemcpyHostToDevice, st));
    CUDA_TRY(c, embed(c->pf_tok, c->embed, c->pf_x, T, d, st));
    for (int l = 0; l < L; ++l) {
      const CUtensorMap* W = &c->pf_wmap[(size_t)l * 4];
      CUDA_TRY(c, rmsnorm_split(c->pf_x, c->attn_norm + (size_t)l * d, c->pf_xh, c->pf_xl, T, d, k.rms_eps, st));
      GemmArgs g{};
      g.err = c->pf_err;
      g.M = qkv_rows; g.N = T; g.K = d; g.epi = EPI_QKV;
      g.q = c->pf_q; g.kcache = c->kcache; g.vcache = c->vcache; g.rope = c->rope;
      g.layer = l; g.hq = hq; g.hk = hk; g.dh = dh; g.max_ctx = k.max_ctx; g.pos0 = p0;
      CUDA_TRY(c, gemm(W[0], c->pf_map_xh, c->pf_map_xl, g, st));
      c->launches += 2;
      if (l == L - 1) break;  // later positions need only this layer's K and V
      AttnArgs at{c->pf_q, c->kcache, c->vcache, c->pf_oh, c->pf_ol, T, p0, l, hq, hk, dh, k.max_ctx};
      CUDA_TRY(c, attention(at, st));
      GemmArgs o{};
      o.err = c->pf_err;
      o.M = d; o.N = T; o.K = hq * dh; o.epi = EPI_RESID; o.x = c->pf_x;
      CUDA_TRY(c, gemm(W[1], c->pf_map_oh, c->pf_map_ol, o, st));
      CUDA_TRY(c, rmsnorm_split(c->pf_x, c->mlp_norm + (size_t)l * d, c->pf_xh, c->pf_xl, T, d, k.rms_eps, st));
      if (moe) {
        // router logits, routing and the expert-sorted rows, then each routed
        // expert over its own rows, the shared expert over all, and the
        // weighted combine into x
        GemmArgs r{};
        r.err = c->pf_err;
        r.M = E; r.N = T; r.K = d; r.epi = EPI_STORE; r.out = c->pf_logits;
        CUDA_TRY(c, gemm(c->pf_rmap[l], c->pf_map_xh, c->pf_map_xl, r, st));
        RouteArgs ra{c->pf_logits, c->pf_sel, c->pf_wt, c->pf_range, c->pf_rowof, c->pf_tokof, c->pf_err, T, E, K};
        CUDA_TRY(c, moe_route(ra, st));
        CUDA_TRY(c, moe_gather(c->pf_tokof, c->pf_xh, c->pf_xl, c->pf_gh, c->pf_gl, T * K, d, st));
        for (int e = 0; e < E; ++e) {
          const CUtensorMap* We = &c->pf_emap[((size_t)l * E + e) * 2];
          GemmArgs u{};
          u.err = c->pf_err;
          u.M = 2 * ffe; u.N = T; u.K = d; u.epi = EPI_SWIGLU; u.h_hi = c->pf_eh; u.h_lo = c->pf_el; u.ff = ffe;
          u.nrange = c->pf_range + 2 * e;
          CUDA_TRY(c, gemm(We[0], c->pf_map_gh, c->pf_map_gl, u, st));
          GemmArgs w{};
          w.err = c->pf_err;
          w.M = d; w.N = T; w.K = ffe; w.epi = EPI_STORE; w.out = c->pf_y; w.nrange = c->pf_range + 2 * e;
          CUDA_TRY(c, gemm(We[1], c->pf_map_eh, c->pf_map_el, w, st));
        }
        if (ff) {
          GemmArgs u{};
          u.err = c->pf_err;
          u.M = 2 * ff; u.N = T; u.K = d; u.epi = EPI_SWIGLU; u.h_hi = c->pf_hh; u.h_lo = c->pf_hl; u.ff = ff;
          CUDA_TRY(c, gemm(W[2], c->pf_map_xh, c->pf_map_xl, u, st));
          GemmArgs w{};
          w.err = c->pf_err;
          w.M = d; w.N = T; w.K = ff; w.epi = EPI_RESID; w.x = c->pf_x;
          CUDA_TRY(c, gemm(W[3], c->pf_map_hh, c->pf_map_hl, w, st));
        }
        CUDA_TRY(c, moe_combine(c->pf_y, c->pf_rowof, c->pf_wt, c->pf_x, T, K, d, st));
        c->launches += 7 + 2 * E + (ff ? 2 : 0);
      } else {
        GemmArgs u{};
        u.err = c->pf_err;
        u.M = 2 * ff; u.N = T; u.K = d; u.epi = EPI_SWIGLU; u.h_hi = c->pf_hh; u.h_lo = c->pf_hl; u.ff = ff;
        CUDA_TRY(c, gemm(W[2], c->pf_map_xh, c->pf_map_xl, u, st));
        GemmArgs w{};
        w.err = c->pf_err;
        w.M = d; w.N = T; w.K = ff; w.epi = EPI_RESID; w.x = c->pf_x;
        CUDA_TRY(c, gemm(W[3], c->pf_map_hh, c->pf_map_hl, w, st));
        c->launches += 5;
      }
    }
    c->launches += 1;
  }
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    c->poisoned = true;
    return fail(c, KIE_ERR_CUDA, "prefill kernels failed: %s", cudaGetErrorString(e));
  }
  int err = 0;
  CUDA_TRY(c, cudaMemcpy(&err, c->pf_err, 4, cudaMemcpyDeviceToHost));
  if (err) {
    c->poisoned = true;
    if (err == 2) return fail(c, KIE_ERR_DEVICE, "prefill routing met a non-finite router logit; context poisoned");
    return fail(c, KIE_ERR_TIMEOUT, "prefill GEMM wait gave up; context poisoned");
  }
  return KIE_OK;
}

extern "C" {

kie_status kie_create(const kie_config* cfg, int device, kie_ctx** out) {
  g_create_error.clear();
  if (!cfg || !out) return fail(nullptr, KIE_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  const kie_config& k = *cfg;
  const bool moe = k.n_experts > 0;
  if (kie_status vs = validate_config(k)) return vs;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return fail(nullptr, KIE_ERR_INVALID_ARG, "no CUDA device %d", device);
  }
  kie_ctx* c = new (std::nothrow) kie_ctx();
  if (!c) return fail(nullptr, KIE_ERR_OOM, "host allocation failed");
  c->cfg = k;
  c->device = device;
  auto bail = [&](kie_status s) {
    g_create_error = c->err;
    kie_destroy(c);
    return s;
  };
  if (cudaSetDevice(device) != cudaSuccess) return bail(fail(c, KIE_ERR_CUDA, "cudaSetDevice failed"));
  cudaDeviceProp prop{};
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess)
    return bail(fail(c, KIE_ERR_CUDA, "cudaGetDeviceProperties failed"));
  if (prop.major < 10) return bail(fail(c, KIE_ERR_CUDA, "device %s is not sm_100", prop.name));
  if (!prop.cooperativeLaunch) return bail(fail(c, KIE_ERR_CUDA, "no cooperative launch support"));
  c->sms = prop.multiProcessorCount;

  const int hq = k.n_heads, hk = k.n_kv_heads, dh = k.head_dim, d = k.d_model;
  c->hbuf = moe ? (k.ffn_shared + k.top_k * k.ffn_expert) : k.ffn;
  // the vector buffer doubles as attention scratch: q of one KV group, the
  // consumer warps' (max, sum, acc) partials and their 32-position score blocks
  // input vectors are stored as two planes (first / second halves of each
  // 8-float chunk), the second at xplane
  const int vmax = std::max({d, hq * dh, c->hbuf});
  c->xplane = ((vmax / 2) + 3) & ~3;
  int vf = std::max(2 * c->xplane,
                    kMaxHeadsPerGroup * dh + kConsumerWarps * kMaxHeadsPerGroup * (dh + 4 + kAttnSub));
  vf = (vf + 3) & ~3;
  c->gbuf_off = vf;           // then d fp16 norm-gain values
  vf += ((d / 2) + 3) & ~3;
  // MoE: then this layer's router columns of the CTA's residual rows, fp16
  // [E][rslice_rows] (for the router partial sums of the output projection)
  const int grid = std::min(c->sms, d);
  c->rslice_off = vf;
  c->rslice_rows = (d + grid - 1) / grid;
  if (moe) vf += ((k.n_experts * c->rslice_rows + 1) / 2 + 3) & ~3;
  c->vec_floats = vf;
  // kRingStages ring stages (two per consumer warp) of the largest size that
  // fits, in 1 KiB steps, at most 16 KiB
  const int fixed = kernel_smem_bytes(vf, 4 * k.n_layers + 1, 0, 0);
  const int optin = (int)prop.sharedMemPerBlockOptin;
  const int ns = kernel_max_stages();
  int sb = std::min(kMaxStageBytes, ((optin - fixed) / ns) & ~1023);
  // a stage holds a weight tile (at least 4 KiB) or one attention sub-block
  // of K or V rows (kAttnSub positions x head_dim fp16)
  if (sb < std::max(4096, kAttnSub * dh * 2))
    return bail(fail(c, KIE_ERR_INVALID_ARG, "shape needs too much shared memory"));
  c->n_stages = ns;
  c->stage_bytes = sb;
  c->smem = kernel_smem_bytes(vf, 4 * k.n_layers + 1, ns, sb);
  if (cudaFuncSetAttribute(kernel_entry(dh, moe), cudaFuncAttributeMaxDynamicSharedMemorySize, c->smem) !=
      cudaSuccess)
    return bail(fail(c, KIE_ERR_CUDA, "cudaFuncSetAttribute(smem=%d) failed: %s", c->smem,
                     cudaGetErrorString(cudaGetLastError())));
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel_entry(dh, moe), kThreads, c->smem) !=
          cudaSuccess ||
      per_sm < 1)
    return bail(fail(c, KIE_ERR_CUDA, "kernel does not fit on an SM (smem %d)", c->smem));
  // one CTA per SM (the ring takes the SM's shared memory), and no more CTAs
  // than residual rows: every CTA publishes residual rows in every layer, and
  // the flagged scratch words are reused layer after layer on the strength of
  // that (a CTA cannot run a layer ahead of one that has not yet read them)
  c->grid = grid;
  if (moe && c->grid > kRouteMaxGrid)
    return bail(fail(c, KIE_ERR_INVALID_ARG, "MoE routing supports at most %d CTAs", kRouteMaxGrid));
  if ((d + c->grid - 1) / c->grid > kMaxOwnRows)
    return bail(fail(c, KIE_ERR_INVALID_ARG, "d_model %d over %d CTAs exceeds %d residual rows per CTA", d,
                     c->grid, kMaxOwnRows));
  c->slots = slots_per_layer(moe ? k.n_experts : 0);

  // attention units cover >= 256 positions and >= T*hk/grid positions each
  const int unit_min = kConsumerWarps * kAttnSub;
  c->max_chunks = std::min((k.max_ctx + unit_min - 1) / unit_min, c->grid / hk + 2);

  kie_status s;
  const size_t kv = (size_t)k.n_layers * hk * k.max_ctx * dh * sizeof(__half);
  if ((s = dalloc(c, &c->kcache, kv)) || (s = dalloc(c, &c->vcache, kv))) return bail(s);
  if ((s = dalloc(c, &c->rope, (size_t)k.max_ctx * (dh / 2) * sizeof(float2)))) return bail(s);
  {
    std::vector<float2> tab((size_t)k.max_ctx * (dh / 2));
    for (int p = 0; p < k.max_ctx; ++p)
      for (int i = 0; i < dh / 2; ++i) {
        const double phi = (double)p * std::pow((double)k.rope_theta, -2.0 * i / dh);
        tab[(size_t)p * (dh / 2) + i] = make_float2((float)std::cos(phi), (float)std::sin(phi));
      }
    if (cudaMemcpy(c->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) !=
        cudaSuccess)
      return bail(fail(c, KIE_ERR_CUDA, "rope table upload failed"));
  }
  if ((s = dalloc(c, &c->tok_dev, (size_t)k.max_ctx * 4)) ||
      (s = dalloc(c, &c->forced_dev, (size_t)k.max_ctx * 4)) ||
      (s = dalloc(c, &c->margins_dev, (size_t)k.max_ctx * 4)))
    return bail(s);
  c->syncblk_bytes = sync_layout(k, c->grid, c->hbuf, c->max_chunks).total;
  if ((s = dalloc(c, &c->syncblk, c->syncblk_bytes))) return bail(s);
  if (cudaMemset(c->syncblk, 0, c->syncblk_bytes) != cudaSuccess)
    return bail(fail(c, KIE_ERR_CUDA, "memset failed"));
  *out = c;
  return KIE_OK;
}

kie_status kie_destroy(kie_ctx* c) {
  if (!c) return KIE_OK;
  cudaSetDevice(c->device);
  for (void* p : c->allocs) cudaFree(p);
  c->allocs.clear();
  delete c;
  return KIE_OK;
}

const char* kie_last_error(const kie_ctx* c) {
  if (!c) return g_create_error.c_str();
  return c->err.c_str();
}

int32_t kie_position(const kie_ctx* c) { return c ? c->pos : -1; }
int32_t kie_pending(const kie_ctx* c) { return c ? c->pending : -1; }

kie_status kie_reset(kie_ctx* c) {
  if (!c) return KIE_ERR_INVALID_ARG;
  c->err.clear();
  cudaSetDevice(c->device);
  cudaError_t e = cudaMemset(c->syncblk, 0, c->syncblk_bytes);
  if (e != cudaSuccess) return fail(c, KIE_ERR_CUDA, "reset memset failed: %s", cudaGetErrorString(e));
  c->pos = 0;
  c->pending = -1;
  c->poisoned = false;
  return KIE_OK;
}

kie_status kie_rewind(kie_ctx* c, int32_t pos, int32_t pending) {
  if (!c) return KIE_ERR_INVALID_ARG;
  c->err.clear();
  if (c->poisoned) return fail(c, KIE_ERR_STATE, "context is poisoned; call kie_reset");
  if (!c->loaded) return fail(c, KIE_ERR_STATE, "weights not loaded");
  if (pos < 0 || pos > c->pos) return fail(c, KIE_ERR_INVALID_ARG, "rewind to %d outside [0, %d]", pos, c->pos);
  if (pending < 0 || pending >= c->cfg.vocab)
    return fail(c, KIE_ERR_INVALID_ARG, "pending token %d outside [0, %d)", pending, c->cfg.vocab);
  c->pos = pos;
  c->pending = pending;
  return KIE_OK;
}

kie_status kie_plan(const kie_config* cfg, int32_t grid, int32_t stage_bytes, kie_plan_info* info,
                    kie_seg_range* ranges, int64_t capacity) {
  g_create_error.clear();
  if (!cfg || !info) return fail(nullptr, KIE_ERR_INVALID_ARG, "null argument");
  if (kie_status vs = validate_config(*cfg)) return vs;
  if (grid < 1) return fail(nullptr, KIE_ERR_INVALID_ARG, "grid %d < 1", grid);
  if (stage_bytes < 4096 || stage_bytes % 16)
    return fail(nullptr, KIE_ERR_INVALID_ARG, "stage_bytes %d: at least 4096 and a multiple of 16", stage_bytes);
  if (cfg && stage_bytes < kAttnSub * cfg->head_dim * 2)
    return fail(nullptr, KIE_ERR_INVALID_ARG, "stage_bytes %d: below one attention sub-block (%d B)", stage_bytes,
                kAttnSub * cfg->head_dim * 2);
  Plan plan;
  if (kie_status ps = make_plan(nullptr, *cfg, grid, stage_bytes, plan)) return ps;
  const int per_cta = cfg->n_layers * plan.slots + 1;
  info->slots = plan.slots;
  info->ranges_per_cta = per_cta;
  info->tape_bytes = (int64_t)plan.tape_bytes;
  for (int i = 0; i < SK_COUNT; ++i)
    info->shapes[i] = kie_seg_shape{plan.shp[i].K, plan.shp[i].g, plan.shp[i].nk, plan.shp[i].kc};
  if (ranges) {
    if (capacity < (int64_t)plan.desc.size())
      return fail(nullptr, KIE_ERR_INVALID_ARG, "ranges holds %lld entries, the plan has %zu",
                  (long long)capacity, plan.desc.size());
    for (size_t i = 0; i < plan.desc.size(); ++i)
      ranges[i] = kie_seg_range{(int64_t)plan.desc[i].off, plan.desc[i].row0, plan.desc[i].nrows};
  }
  return KIE_OK;
}

kie_status kie_get_info(const kie_ctx* c, kie_info* info) {
  if (!c || !info) return KIE_ERR_INVALID_ARG;
  if (!c->loaded) return KIE_ERR_STATE;
  const kie_config& k = c->cfg;
  info->grid = c->grid;
  info->threads = kThreads;
  info->n_stages = c->n_stages;
  info->stage_bytes = c->stage_bytes;
  info->smem_bytes = c->smem;
  info->barriers_per_token = 1;
  info->stream_bytes = c->stream_bytes;
  info->kv_bytes_per_pos = 2LL * k.n_layers * k.n_kv_heads * k.head_dim * 2;
  info->resident_bytes = (int64_t)c->tape_bytes;
  info->launches = c->launches;
  return KIE_OK;
}

kie_status kie_load_weights(kie_ctx* c, const kie_tensor* tensors, int n, void* stream) {
  if (!c) return KIE_ERR_INVALID_ARG;
  c->err.clear();
  if (!tensors || n <= 0) return fail(c, KIE_ERR_INVALID_ARG, "no tensors");
  cudaSetDevice(c->device);
  cudaStream_t st = (cudaStream_t)stream;
  const kie_config& k = c->cfg;
  const bool moe = k.n_experts > 0;
  const int d = k.d_model, hq = k.n_heads, hk = k.n_kv_heads, dh = k.head_dim, L = k.n_layers;

  // expected tensors
  std::map<std::string, std::pair<int64_t, int64_t>> want;
  auto W = [&](const std::string& nm, int64_t r, int64_t cc) { want[nm] = {r, cc}; };
  W("embed", k.vocab, d);
  W("lm_head", k.vocab, d);
  W("final_norm", d, 1);
  for (int l = 0; l < L; ++l) {
    const std::string p = "layers." + std::to_string(l) + ".";
    W(p + "attn_norm", d, 1);
    W(p + "mlp_norm", d, 1);
    W(p + "wq", (int64_t)hq * dh, d);
    W(p + "wk", (int64_t)hk * dh, d);
    W(p + "wv", (int64_t)hk * dh, d);
    W(p + "wo", d, (int64_t)hq * dh);
    if (!moe) {
      W(p + "w_gate", k.ffn, d);
      W(p + "w_up", k.ffn, d);
      W(p + "w_down", d, k.ffn);
    } else {
      W(p + "router", k.n_experts, d);
      for (int e = 0; e < k.n_experts; ++e) {
        const std::string q = p + "experts." + std::to_string(e) + ".";
        W(q + "w_gate", k.ffn_expert, d);
        W(q + "w_up", k.ffn_expert, d);
        W(q + "w_down", d, k.ffn_expert);
      }
      if (k.ffn_shared) {  // a model without a shared expert has no shared tensors
        W(p + "shared.w_gate", k.ffn_shared, d);
        W(p + "shared.w_up", k.ffn_shared, d);
        W(p + "shared.w_down", d, k.ffn_shared);
      }
    }
  }
  std::map<std::string, Tensor> got;
  for (int i = 0; i < n; ++i) {
    const kie_tensor& t = tensors[i];
    if (!t.name || !t.data) return fail(c, KIE_ERR_INVALID_ARG, "tensor %d has a null name or data", i);
    auto it = want.find(t.name);
    if (it == want.end()) return fail(c, KIE_ERR_INVALID_ARG, "unexpected tensor '%s'", t.name);
    if (got.count(t.name)) return fail(c, KIE_ERR_INVALID_ARG, "tensor '%s' given twice", t.name);
    int64_t r = t.shape[0], cc = t.shape[1];
    const bool vec = it->second.second == 1;
    if (vec && r == 1 && cc == it->second.first) std::swap(r, cc);
    if (r != it->second.first || cc != it->second.second)
      return fail(c, KIE_ERR_INVALID_ARG, "tensor '%s' has shape [%lld, %lld], expected [%lld, %lld]",
                  t.name, (long long)t.shape[0], (long long)t.shape[1], (long long)it->second.first,
                  (long long)it->second.second);
    if (t.on_device && ptr_device(t.data) != c->device)
      return fail(c, KIE_ERR_INVALID_ARG, "tensor '%s' marked on_device but is not memory of device %d", t.name,
                  c->device);
    if (t.on_device && (reinterpret_cast<uintptr_t>(t.data) & 15))
      return fail(c, KIE_ERR_INVALID_ARG, "device tensor '%s' is not 16-byte aligned", t.name);
    got[t.name] = Tensor{t.data, r, cc, t.on_device != 0};
  }
  for (auto& kv : want)
    if (!got.count(kv.first)) return fail(c, KIE_ERR_INVALID_ARG, "missing tensor '%s'", kv.first.c_str());

  // release a previous load
  dfree(c, c->tape); c->tape = nullptr;
  dfree(c, c->desc); c->desc = nullptr;
  dfree(c, c->embed); c->embed = nullptr;
  dfree(c, c->attn_norm); c->attn_norm = nullptr;
  dfree(c, c->mlp_norm); c->mlp_norm = nullptr;
  dfree(c, c->final_norm); c->final_norm = nullptr;
  dfree(c, c->router); c->router = nullptr;
  c->loaded = false;

  // stage host tensors on the device (device tensors are read in place)
  size_t stage_bytes = 0;
  std::map<std::string, size_t> soff;
  for (auto& kv : got)
    if (!kv.second.on_dev) {
      soff[kv.first] = stage_bytes;
      stage_bytes += ((size_t)kv.second.rows * kv.second.cols * 2 + 255) & ~(size_t)255;
    }
  unsigned char* staging = nullptr;
  kie_status s;
  if (stage_bytes && (s = dalloc(c, &staging, stage_bytes))) return s;
  std::map<std::string, const unsigned char*> dptr;
  for (auto& kv : got) {
    if (kv.second.on_dev) {
      dptr[kv.first] = static_cast<const unsigned char*>(kv.second.data);
    } else {
      unsigned char* dst = staging + soff[kv.first];
      const size_t bytes = (size_t)kv.second.rows * kv.second.cols * 2;
      cudaError_t e = cudaMemcpyAsync(dst, kv.second.data, bytes, cudaMemcpyHostToDevice, st);
      if (e != cudaSuccess) {
        dfree(c, staging);
        return fail(c, KIE_ERR_CUDA, "upload of '%s' failed: %s", kv.first.c_str(), cudaGetErrorString(e));
      }
      dptr[kv.first] = dst;
    }
  }

  // segment shapes, row assignment and tape offsets
  const int ffs = k.ffn_shared, ffe = k.ffn_expert;
  const int G = c->grid;
  Plan plan;
  if ((s = make_plan(c, k, G, c->stage_bytes, plan))) {
    dfree(c, staging);
    return s;
  }
  for (int i = 0; i < SK_COUNT; ++i) c->shp[i] = plan.shp[i];
  c->lm_rows = 0;
  for (int ci = 0; ci < G; ++ci)
    c->lm_rows = std::max(c->lm_rows, plan.desc[(size_t)ci * (L * c->slots + 1) + (size_t)L * c->slots].nrows);
  auto kind_of = [&](int l, int slot) -> int { return ::kind_of(k, l, slot); };
  const int per_cta = L * c->slots + 1;
  const std::vector<SegDesc>& desc = plan.desc;
  c->tape_bytes = plan.tape_bytes;
  if ((s = dalloc(c, &c->tape, c->tape_bytes))) {
    dfree(c, staging);
    return s;
  }

  // row-copy list: virtual row -> source row pointer
  auto rowptr = [&](int l, int slot, int row) -> const unsigned char* {
    const int kind = kind_of(l, slot);
    const std::string p = "layers." + std::to_string(l) + ".";
    switch (kind) {
      case SK_QKV: {
        // virtual rows of a head run (0, dh/2, 1, dh/2 + 1, ...) so RoPE pairs are adjacent
        const int H = row / dh, v = row % dh;
        const int dim = (v & 1) ? v / 2 + dh / 2 : v / 2;
        if (H < hq) return dptr[p + "wq"] + ((size_t)H * dh + dim) * d * 2;
        if (H < hq + hk) return dptr[p + "wk"] + ((size_t)(H - hq) * dh + dim) * d * 2;
        return dptr[p + "wv"] + ((size_t)(H - hq - hk) * dh + dim) * d * 2;
      }
      case SK_O: return dptr[p + "wo"] + (size_t)row * hq * dh * 2;
      case SK_GU: return dptr[p + ((row & 1) ? "w_up" : "w_gate")] + (size_t)(row / 2) * d * 2;
      case SK_DOWN: return dptr[p + "w_down"] + (size_t)row * k.ffn * 2;
      case SK_SGU: return dptr[p + ((row & 1) ? "shared.w_up" : "shared.w_gate")] + (size_t)(row / 2) * d * 2;
      case SK_SDOWN: return dptr[p + "shared.w_down"] + (size_t)row * ffs * 2;
      case SK_EGU: {
        const int e = slot - 4;
        const std::string q = p + "experts." + std::to_string(e) + ".";
        return dptr[q + ((row & 1) ? "w_up" : "w_gate")] + (size_t)(row / 2) * d * 2;
      }
      case SK_EDOWN: {
        const int e = slot - 4 - k.n_experts;
        return dptr[p + "experts." + std::to_string(e) + ".w_down"] + (size_t)row * ffe * 2;
      }
      default: return dptr["lm_head"] + (size_t)row * d * 2;
    }
  };
  // cache the string lookups per (layer, slot) by resolving row 0 and 1 bases lazily:
  // the list is built layer by layer to bound host memory.
  std::vector<unsigned long long> hsrc, hdst;
  std::vector<int> hn;
  unsigned long long* dsrc = nullptr;
  unsigned long long* ddst = nullptr;
  int* dn = nullptr;
  size_t cap = 0;
  auto flush = [&]() -> kie_status {
    const size_t m = hsrc.size();
    if (!m) return KIE_OK;
    if (m > cap) {
      dfree(c, dsrc); dfree(c, ddst); dfree(c, dn);
      dsrc = ddst = nullptr; dn = nullptr;
      cap = m;
      kie_status s2;
      if ((s2 = dalloc(c, &dsrc, m * 8)) || (s2 = dalloc(c, &ddst, m * 8)) || (s2 = dalloc(c, &dn, m * 4)))
        return s2;
    }
    CUDA_TRY(c, cudaMemcpyAsync(dsrc, hsrc.data(), m * 8, cudaMemcpyHostToDevice, st));
    CUDA_TRY(c, cudaMemcpyAsync(ddst, hdst.data(), m * 8, cudaMemcpyHostToDevice, st));
    CUDA_TRY(c, cudaMemcpyAsync(dn, hn.data(), m * 4, cudaMemcpyHostToDevice, st));
    const int blocks = (int)std::min<size_t>((m + 7) / 8, 4096);
    pack_rows_kernel<<<blocks, 256, 0, st>>>(dsrc, ddst, dn, (long long)m);
    CUDA_TRY(c, cudaGetLastError());
    c->launches++;
    CUDA_TRY(c, cudaStreamSynchronize(st));  // host vectors are reused
    hsrc.clear(); hdst.clear(); hn.clear();
    return KIE_OK;
  };
  kie_status ps = KIE_OK;
  for (int l = 0; l <= L && ps == KIE_OK; ++l) {
    const int nsl = (l == L) ? 1 : c->slots;
    for (int slot = 0; slot < nsl; ++slot) {
      const SegShape& sh = c->shp[kind_of(l, slot)];
      // resolve two base pointers per slot once (even/odd rows for GU kinds)
      for (int ci = 0; ci < G; ++ci) {
        const SegDesc& sd = desc[(size_t)ci * per_cta + (size_t)l * c->slots + slot];
        const int ngroups = (sd.nrows + sh.g - 1) / sh.g;
        for (int gi = 0; gi < ngroups; ++gi) {
          const int gp = std::min(sh.g, sd.nrows - gi * sh.g);
          for (int kj = 0; kj < sh.nk; ++kj) {
            for (int r = 0; r < gp; ++r) {
              const int row = sd.row0 + gi * sh.g + r;
              const unsigned char* src = rowptr(l, slot, row) + (size_t)kj * sh.kc * 2;
              unsigned char* dst = c->tape + sd.off + (size_t)gi * sh.g * sh.K * 2 +
                                   (size_t)kj * gp * sh.kc * 2 + (size_t)r * sh.kc * 2;
              hsrc.push_back((unsigned long long)src);
              hdst.push_back((unsigned long long)dst);
              hn.push_back(sh.kc / 8);
            }
          }
        }
      }
    }
    ps = flush();
  }
  if (ps != KIE_OK) {
    dfree(c, staging);
    return ps;
  }
  // the prefill's row-major copies of the layer matrices in the packed row
  // orders (slots 0-3: q/k/v, o, and the dense or shared-expert gate/up and
  // down; MoE: the routed experts and the router as well)
  for (int i = 0; i < 4; ++i) { dfree(c, c->pf_w[i]); c->pf_w[i] = nullptr; }
  for (int i = 0; i < 2; ++i) { dfree(c, c->pf_we[i]); c->pf_we[i] = nullptr; }
  dfree(c, c->pf_router); c->pf_router = nullptr;
  c->pf_ready = false;
  {
    const int fw = moe ? ffs : k.ffn;
    const int prow[4] = {(hq + 2 * hk) * dh, d, 2 * fw, d};
    const int pk[4] = {d, hq * dh, d, fw};
    for (int m = 0; m < 4 && ps == KIE_OK; ++m) {
      if (m >= 2 && fw == 0) break;  // no shared expert
      if ((ps = dalloc(c, &c->pf_w[m], (size_t)L * prow[m] * pk[m] * 2))) break;
      for (int l = 0; l < L && ps == KIE_OK; ++l) {
        for (int r = 0; r < prow[m]; ++r) {
          hsrc.push_back((unsigned long long)rowptr(l, m, r));
          hdst.push_back((unsigned long long)(c->pf_w[m] + ((size_t)l * prow[m] + r) * pk[m]));
          hn.push_back(pk[m] / 8);
        }
        ps = flush();
      }
    }
    if (moe && ps == KIE_OK) {
      const int E = k.n_experts;
      const int erow[2] = {2 * ffe, d}, ek[2] = {d, ffe};
      for (int m = 0; m < 2 && ps == KIE_OK; ++m) {
        if ((ps = dalloc(c, &c->pf_we[m], (size_t)L * E * erow[m] * ek[m] * 2))) break;
        for (int l = 0; l < L && ps == KIE_OK; ++l) {
          for (int e = 0; e < E; ++e)
            for (int r = 0; r < erow[m]; ++r) {
              hsrc.push_back((unsigned long long)rowptr(l, 4 + m * E + e, r));
              hdst.push_back((unsigned long long)(c->pf_we[m] + (((size_t)l * E + e) * erow[m] + r) * ek[m]));
              hn.push_back(ek[m] / 8);
            }
          ps = flush();
        }
      }
      // the router, zero rows past E up to a whole GEMM tile
      c->pf_epad = (E + kie::pf::kBM - 1) / kie::pf::kBM * kie::pf::kBM;
      if (ps == KIE_OK && (ps = dalloc(c, &c->pf_router, (size_t)L * c->pf_epad * d * 2)) == KIE_OK) {
        CUDA_TRY(c, cudaMemsetAsync(c->pf_router, 0, (size_t)L * c->pf_epad * d * 2, st));
        for (int l = 0; l < L; ++l)
          CUDA_TRY(c, cudaMemcpyAsync(c->pf_router + (size_t)l * c->pf_epad * d,
                                      dptr["layers." + std::to_string(l) + ".router"], (size_t)E * d * 2,
                                      cudaMemcpyDeviceToDevice, st));
      }
    }
    if (ps != KIE_OK) {
      dfree(c, staging);
      return ps;
    }
  }
  dfree(c, dsrc); dfree(c, ddst); dfree(c, dn);

  // descriptors and the small tensors kept outside the tape
  if ((s = dalloc(c, &c->desc, desc.size() * sizeof(SegDesc)))) return s;
  CUDA_TRY(c, cudaMemcpyAsync(c->desc, desc.data(), desc.size() * sizeof(SegDesc),
                              cudaMemcpyHostToDevice, st));
  if ((s = dalloc(c, &c->embed, (size_t)k.vocab * d * 2)) ||
      (s = dalloc(c, &c->attn_norm, (size_t)L * d * 2)) || (s = dalloc(c, &c->mlp_norm, (size_t)L * d * 2)) ||
      (s = dalloc(c, &c->final_norm, (size_t)d * 2)))
    return s;
  CUDA_TRY(c, cudaMemcpyAsync(c->embed, dptr["embed"], (size_t)k.vocab * d * 2, cudaMemcpyDeviceToDevice, st));
  CUDA_TRY(c, cudaMemcpyAsync(c->final_norm, dptr["final_norm"], (size_t)d * 2, cudaMemcpyDeviceToDevice, st));
  for (int l = 0; l < L; ++l) {
    const std::string p = "layers." + std::to_string(l) + ".";
    CUDA_TRY(c, cudaMemcpyAsync(c->attn_norm + (size_t)l * d, dptr[p + "attn_norm"], (size_t)d * 2,
                                cudaMemcpyDeviceToDevice, st));
    CUDA_TRY(c, cudaMemcpyAsync(c->mlp_norm + (size_t)l * d, dptr[p + "mlp_norm"], (size_t)d * 2,
                                cudaMemcpyDeviceToDevice, st));
  }
  if (moe) {
    if ((s = dalloc(c, &c->router, (size_t)L * k.n_experts * d * 2))) return s;
    for (int l = 0; l < L; ++l)
      CUDA_TRY(c, cudaMemcpyAsync(c->router + (size_t)l * k.n_experts * d,
                                  dptr["layers." + std::to_string(l) + ".router"],
                                  (size_t)k.n_experts * d * 2, cudaMemcpyDeviceToDevice, st));
  }
  CUDA_TRY(c, cudaStreamSynchronize(st));
  dfree(c, staging);

  // algorithmic weight bytes streamed per decoded token
  int64_t sb = 0;
  const int64_t qkvb = (int64_t)(hq + 2 * hk) * dh * d * 2, ob = (int64_t)d * hq * dh * 2;
  if (!moe) {
    sb = L * (qkvb + ob + 3LL * k.ffn * d * 2);
  } else {
    sb = L * (qkvb + ob + (int64_t)k.n_experts * d * 2 + 3LL * ffs * d * 2 + k.top_k * 3LL * ffe * d * 2);
  }
  sb += (int64_t)k.vocab * d * 2 + (2LL * L + 1) * d * 2 + (int64_t)d * 2;
  c->stream_bytes = sb;
  {
    kie_status s2 = prefill_setup(c);
    if (s2 != KIE_OK) return s2;
  }
  c->loaded = true;
  c->pos = 0;
  c->pending = -1;
  c->poisoned = false;
  return KIE_OK;
}

}  // extern "C"

namespace {

struct Run {
  int first_token, n_steps, lm_from_step;
  const int* forced;
  int* out;
  float* logits;
  float* margins;
  uint32_t timeout_ms;
  int fault_cta, fault_barrier;
  uint64_t* trace;
  int trace_cap;
  float temperature = 0.f, top_p = 1.f;
  int top_k = 0;
  uint64_t seed = 0;
};

// The kernel's parameter block for run `r`, with the per-launch scratch (the
// region cleared before every launch: control block and flagged words) at
// `sync_base`. Both entry points that launch the kernel build their
// parameters here.
Params make_params(const kie_ctx* c, const Run& r, unsigned char* sync_base) {
  const kie_config& k = c->cfg;
  Params P{};
  P.L = k.n_layers; P.d = k.d_model; P.hq = k.n_heads; P.hk = k.n_kv_heads; P.dh = k.head_dim;
  P.ff = k.ffn; P.V = k.vocab; P.E = k.n_experts; P.top_k = k.top_k; P.ffe = k.ffn_expert;
  P.ffs = k.ffn_shared; P.max_ctx = k.max_ctx; P.eps = k.rms_eps;
  P.qkv_rows = (k.n_heads + 2 * k.n_kv_heads) * k.head_dim;
  P.slots = c->slots;
  P.tape = c->tape; P.desc = c->desc;
  for (int i = 0; i < SK_COUNT; ++i) P.shp[i] = c->shp[i];
  P.embed = c->embed; P.attn_norm = c->attn_norm; P.mlp_norm = c->mlp_norm;
  P.final_norm = c->final_norm; P.router = c->router;
  P.kcache = c->kcache; P.vcache = c->vcache; P.rope = c->rope;
  set_sync_params(P, sync_base, sync_layout(k, c->grid, c->hbuf, c->max_chunks));
  P.max_chunks = c->max_chunks;
  P.pos0 = c->pos; P.n_steps = r.n_steps; P.first_token = r.first_token; P.lm_from_step = r.lm_from_step;
  P.forced = r.forced; P.out_tokens = r.out; P.logits_out = r.logits; P.margins_out = r.margins;
  P.timeout_ns = (unsigned long long)(r.timeout_ms ? r.timeout_ms : 1000u) * 1000000ull;
  P.fault_cta = r.fault_cta; P.fault_barrier = r.fault_barrier;
  P.trace = reinterpret_cast<unsigned long long*>(r.trace); P.trace_cap = r.trace_cap;
  P.n_stages = c->n_stages; P.stage_bytes = c->stage_bytes; P.vec_floats = c->vec_floats;
  P.xplane = c->xplane;
  P.gbuf_off = c->gbuf_off;
  P.rslice_off = c->rslice_off;
  P.rslice_rows = c->rslice_rows;
  P.samp_temp = r.temperature; P.samp_p = r.top_p; P.samp_k = r.top_k; P.samp_seed = r.seed;
  P.fsamp = c->fsamp;
  P.lm_logits = c->lm_logits;
  P.lm_rows = c->lm_rows;
  return P;
}

// Clear the per-launch scratch at `sync_base` (`sync_bytes`), launch the
// kernel for run `r`, wait for it and read its error record. On success the
// pending token becomes the kernel's last one (position bookkeeping is the
// caller's).
kie_status launch_on(kie_ctx* c, const Run& r, unsigned char* sync_base, size_t sync_bytes, cudaStream_t st) {
  Params P = make_params(c, r, sync_base);
  CUDA_TRY(c, cudaMemsetAsync(sync_base, 0, sync_bytes, st));
  if (r.temperature > 0.f) CUDA_TRY(c, cudaMemsetAsync(c->fsamp, 0, c->fsamp_bytes, st));
  void* args[] = {&P};
  cudaError_t e = cudaLaunchCooperativeKernel(kernel_entry(c->cfg.head_dim, c->cfg.n_experts > 0), dim3(c->grid), dim3(kThreads), args,
                                              (size_t)c->smem, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(c, KIE_ERR_CUDA, "cooperative launch failed: %s", cudaGetErrorString(e));
  }
  c->launches++;
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    c->poisoned = true;
    return fail(c, KIE_ERR_CUDA, "decode kernel failed: %s", cudaGetErrorString(e));
  }
  Ctrl ctl{};
  CUDA_TRY(c, cudaMemcpy(&ctl, sync_base, sizeof(Ctrl), cudaMemcpyDeviceToHost));
  if (ctl.err) {
    c->poisoned = true;
    static const char* where[] = {"?", "grid barrier", "ring stage (full)", "ring stage (empty)",
                                  "expert routing hand-off", "device check", "flagged input wait",
                                  "ring tile larger than a stage"};
    const int w = (ctl.err_where >= 1 && ctl.err_where <= 7) ? ctl.err_where : 0;
    return fail(c, (kie_status)ctl.err, "device %s at %s (cta %d, step %d); context poisoned",
                ctl.err == KIE_ERR_TIMEOUT ? "timeout" : "check failed", where[w], ctl.err_cta,
                ctl.err_step);
  }
  c->pending = ctl.final_token;
  return KIE_OK;
}

// A launch with the context's own scratch.
kie_status launch(kie_ctx* c, const Run& r, cudaStream_t st) {
  return launch_on(c, r, c->syncblk, c->syncblk_bytes, st);
}

}  // namespace

extern "C" {

kie_status kie_prefill(kie_ctx* c, const int32_t* tokens, int n, void* stream) {
  if (!c) return KIE_ERR_INVALID_ARG;
  c->err.clear();
  if (c->poisoned) return fail(c, KIE_ERR_STATE, "context is poisoned; call kie_reset");
  if (!c->loaded) return fail(c, KIE_ERR_STATE, "weights not loaded");
  if (n < 0 || (n > 0 && !tokens)) return fail(c, KIE_ERR_INVALID_ARG, "bad token array");
  if (n == 0) return KIE_OK;
  if (is_device_ptr(tokens)) return fail(c, KIE_ERR_INVALID_ARG, "prefill tokens must be host memory");
  for (int i = 0; i < n; ++i)
    if (tokens[i] < 0 || tokens[i] >= c->cfg.vocab)
      return fail(c, KIE_ERR_INVALID_ARG, "token %d at index %d outside [0, %d)", tokens[i], i, c->cfg.vocab);
  std::vector<int32_t> seq;
  if (c->pending >= 0) seq.push_back(c->pending);
  for (int i = 0; i + 1 < n; ++i) seq.push_back(tokens[i]);
  if ((int64_t)c->pos + (int64_t)seq.size() > c->cfg.max_ctx)
    return fail(c, KIE_ERR_CONTEXT_FULL, "position %d + %zu tokens exceeds max_ctx %d", c->pos, seq.size(),
                c->cfg.max_ctx);
  cudaSetDevice(c->device);
  cudaStream_t st = (cudaStream_t)stream;
  const int32_t new_pending = tokens[n - 1];
  const int32_t pos_before = c->pos, pend_before = c->pending;
  if (!c->pf_ready) return fail(c, KIE_ERR_STATE, "the prompt path is not set up (load weights first)");
  // the chunked tensor-core prefill
  kie_status s = prefill_tc(c, seq, st);
  if (s != KIE_OK) {
    if (!c->poisoned) { c->pos = pos_before; c->pending = pend_before; }
    return s;
  }
  c->pos += (int32_t)seq.size();
  c->pending = new_pending;
  return KIE_OK;
}

kie_status kie_decode(kie_ctx* c, int n, int32_t* out_tokens, const kie_decode_opts* opts, void* stream) {
  if (!c) return KIE_ERR_INVALID_ARG;
  c->err.clear();
  if (c->poisoned) return fail(c, KIE_ERR_STATE, "context is poisoned; call kie_reset");
  if (!c->loaded) return fail(c, KIE_ERR_STATE, "weights not loaded");
  if (n < 0) return fail(c, KIE_ERR_INVALID_ARG, "negative token count");
  if (n == 0) return KIE_OK;
  if (!out_tokens) return fail(c, KIE_ERR_INVALID_ARG, "out_tokens is null");
  if (c->pending < 0) return fail(c, KIE_ERR_STATE, "no pending token: prefill first");
  if ((int64_t)c->pos + n > c->cfg.max_ctx)
    return fail(c, KIE_ERR_CONTEXT_FULL, "position %d + %d tokens exceeds max_ctx %d", c->pos, n, c->cfg.max_ctx);
  kie_decode_opts o{};
  o.fault_cta = -1;
  o.fault_barrier = -1;
  if (opts) o = *opts;
  if (o.trace_out && o.trace_cap <= 0) return fail(c, KIE_ERR_INVALID_ARG, "trace_cap must be > 0");
  if (!(o.temperature >= 0.f) || o.temperature > 1e6f)
    return fail(c, KIE_ERR_INVALID_ARG, "temperature must be >= 0");
  if (o.temperature > 0.f) {
    if (o.top_k < 1 || o.top_k > kSampleK)
      return fail(c, KIE_ERR_INVALID_ARG, "sampling needs 1 <= top_k <= %d (got %d)", kSampleK, o.top_k);
    if (!(o.top_p > 0.f && o.top_p <= 1.f)) return fail(c, KIE_ERR_INVALID_ARG, "top_p must be in (0, 1]");
    if (c->grid > kSampleMaxGrid) return fail(c, KIE_ERR_INVALID_ARG, "sampling supports at most %d CTAs", kSampleMaxGrid);
    if (!c->fsamp) {
      c->fsamp_bytes = ((size_t)c->grid * 2 * kSampleK + 4) * 8;
      kie_status s0 = dalloc(c, &c->fsamp, c->fsamp_bytes);
      if (s0) return s0;
    }
    if (!c->lm_logits) {
      kie_status s0 = dalloc(c, &c->lm_logits, (size_t)c->grid * std::max(1, c->lm_rows) * 4);
      if (s0) return s0;
    }
  }
  if (o.trace_out && ptr_device(o.trace_out) != c->device)
    return fail(c, KIE_ERR_INVALID_ARG, "trace_out must be memory of device %d", c->device);
  {
    kie_status ps;
    if ((ps = check_own_device(c, out_tokens, "out_tokens")) ||
        (ps = check_own_device(c, o.forced_tokens, "forced_tokens")) ||
        (ps = check_own_device(c, o.logits_out, "logits_out")) ||
        (ps = check_own_device(c, o.margins_out, "margins_out")))
      return ps;
  }
  cudaSetDevice(c->device);
  cudaStream_t st = (cudaStream_t)stream;
  const int V = c->cfg.vocab;

  const int* forced = nullptr;
  if (o.forced_tokens) {
    std::vector<int32_t> f(n);
    if (is_device_ptr(o.forced_tokens)) {
      CUDA_TRY(c, cudaMemcpyAsync(f.data(), o.forced_tokens, (size_t)n * 4, cudaMemcpyDeviceToHost, st));
      CUDA_TRY(c, cudaStreamSynchronize(st));
    } else
      std::memcpy(f.data(), o.forced_tokens, (size_t)n * 4);
    for (int i = 0; i < n; ++i)
      if (f[i] < -1 || f[i] >= V)
        return fail(c, KIE_ERR_INVALID_ARG, "forced token %d at step %d outside [-1, %d)", f[i], i, V);
    CUDA_TRY(c, cudaMemcpyAsync(c->forced_dev, f.data(), (size_t)n * 4, cudaMemcpyHostToDevice, st));
    forced = c->forced_dev;
  }
  const bool out_dev = is_device_ptr(out_tokens);
  float* logits = nullptr;
  float* logits_tmp = nullptr;
  if (o.logits_out) {
    if (is_device_ptr(o.logits_out)) {
      logits = o.logits_out;
    } else {
      kie_status s = dalloc(c, &logits_tmp, (size_t)n * V * 4);
      if (s) return s;
      logits = logits_tmp;
    }
  }
  float* margins = nullptr;
  if (o.margins_out) margins = is_device_ptr(o.margins_out) ? o.margins_out : c->margins_dev;
  Run r{c->pending, n, 0, forced, out_dev ? out_tokens : c->tok_dev, logits, margins, o.timeout_ms,
        o.fault_cta, o.fault_barrier, o.trace_out, o.trace_cap, o.temperature, o.top_p, o.top_k, o.seed};
  kie_status s = launch(c, r, st);
  if (s == KIE_OK) {
    if (!out_dev) {
      cudaError_t e = cudaMemcpyAsync(out_tokens, c->tok_dev, (size_t)n * 4, cudaMemcpyDefault, st);
      if (e == cudaSuccess && logits_tmp)
        e = cudaMemcpyAsync(o.logits_out, logits_tmp, (size_t)n * V * 4, cudaMemcpyDefault, st);
      if (e == cudaSuccess && o.margins_out && margins == c->margins_dev)
        e = cudaMemcpyAsync(o.margins_out, margins, (size_t)n * 4, cudaMemcpyDefault, st);
      if (e == cudaSuccess) e = cudaStreamSynchronize(st);
      if (e != cudaSuccess) s = fail(c, KIE_ERR_CUDA, "result copy failed: %s", cudaGetErrorString(e));
    } else {
      cudaError_t e = cudaSuccess;
      if (logits_tmp) e = cudaMemcpyAsync(o.logits_out, logits_tmp, (size_t)n * V * 4, cudaMemcpyDefault, st);
      if (e == cudaSuccess && o.margins_out && margins == c->margins_dev)
        e = cudaMemcpyAsync(o.margins_out, margins, (size_t)n * 4, cudaMemcpyDefault, st);
      if (e == cudaSuccess) e = cudaStreamSynchronize(st);
      if (e != cudaSuccess) s = fail(c, KIE_ERR_CUDA, "result copy failed: %s", cudaGetErrorString(e));
    }
    if (s == KIE_OK) c->pos += n;
  }
  if (logits_tmp) dfree(c, logits_tmp);
  return s;
}

}  // extern "C"

// ------------------------------------------------------------ no-allocation decode
//
// kie_decode_static runs the same persistent decode kernel as kie_decode, but
// the kernel's per-launch scratch (residual stream, q/k/v, attention output,
// FFN hidden vector, attention chunk records, MoE router partials, per-CTA
// argmax candidates, control block) lives in this file-scope device array instead of
// buffers allocated with the context. The call itself allocates nothing.

namespace {

constexpr size_t kStaticScratchBytes = 512u << 10;  // 512 KiB per device
constexpr int kMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

std::mutex g_static_mu;
unsigned char* g_static_ptr[kMaxDevices] = {};

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

struct StaticLayout {
  size_t sync, sync_bytes, total;
};

StaticLayout static_layout(const kie_ctx* c) {
  const kie_config& k = c->cfg;
  StaticLayout L{};
  size_t off = 0;
  L.sync = off;
  L.sync_bytes = sync_layout(k, c->grid, c->hbuf, c->max_chunks).total;
  off += align256(L.sync_bytes);
  L.total = off;
  return L;
}

}  // namespace

extern "C" kie_status kie_decode_static(kie_ctx* c, int n, int32_t* out_tokens, void* stream) {
  if (!c) return KIE_ERR_INVALID_ARG;
  c->err.clear();
  if (c->poisoned) return fail(c, KIE_ERR_STATE, "context is poisoned; call kie_reset");
  if (!c->loaded) return fail(c, KIE_ERR_STATE, "weights not loaded");
  const StaticLayout lay = static_layout(c);
  if (lay.total > kStaticScratchBytes)
    return fail(c, KIE_ERR_INVALID_ARG, "this model needs %zu bytes of scratch; the static area holds %zu",
                lay.total, kStaticScratchBytes);
  if (c->device < 0 || c->device >= kMaxDevices) return fail(c, KIE_ERR_INVALID_ARG, "device %d out of range", c->device);
  if (n < 0) return fail(c, KIE_ERR_INVALID_ARG, "negative token count");
  if (n == 0) return KIE_OK;
  if (!out_tokens || ptr_device(out_tokens) != c->device)
    return fail(c, KIE_ERR_INVALID_ARG, "out_tokens must be memory of device %d", c->device);
  if (c->pending < 0) return fail(c, KIE_ERR_STATE, "no pending token: prefill first");
  if ((int64_t)c->pos + n > c->cfg.max_ctx)
    return fail(c, KIE_ERR_CONTEXT_FULL, "position %d + %d tokens exceeds max_ctx %d", c->pos, n, c->cfg.max_ctx);
  CUDA_TRY(c, cudaSetDevice(c->device));
  unsigned char* base = nullptr;
  {
    // once per device, with that device current: the array's device address
    std::lock_guard<std::mutex> g(g_static_mu);
    if (!g_static_ptr[c->device]) {
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(c, KIE_ERR_CUDA, "cudaGetSymbolAddress(static scratch) failed: %s", cudaGetErrorString(e));
      }
      g_static_ptr[c->device] = static_cast<unsigned char*>(p);
    }
    base = g_static_ptr[c->device];
  }
  cudaStream_t st = (cudaStream_t)stream;
  // the array keeps the previous call's contents: the barrier counter, the
  // abort flag and the flagged words' epochs must start at zero, which
  // launch_on's clear of the sync region ensures
  const Run r{c->pending, n, 0, nullptr, out_tokens, nullptr, nullptr, 0, -1, -1, nullptr, 0};
  kie_status s = launch_on(c, r, base + lay.sync, lay.sync_bytes, st);
  if (s != KIE_OK) return s;
  c->pos += n;
  return KIE_OK;
}
