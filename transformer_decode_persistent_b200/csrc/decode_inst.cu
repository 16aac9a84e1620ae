// Instantiations of the decode kernel (monokernel.cuh), one per head_dim and
// FFN kind, and the host-side accessors the launcher uses.
//
// The build compiles this file once per combination (-DKIE_DH=128|64
// -DKIE_MOE=0|1, in parallel); compiled with neither macro it instantiates all
// four in one translation unit. kernel_smem_bytes and kernel_max_stages are
// defined in exactly one of the objects.
#include "monokernel.cuh"

namespace kie {

#define KIE_DECODE_ENTRY(DH, MOE)                                          \
  const void* kernel_entry_##DH##_##MOE() {                                \
    return reinterpret_cast<const void*>(&decode_kernel<DH, (MOE) != 0>); \
  }

#if !defined(KIE_DH)
KIE_DECODE_ENTRY(128, 0)
KIE_DECODE_ENTRY(128, 1)
KIE_DECODE_ENTRY(64, 0)
KIE_DECODE_ENTRY(64, 1)
#define KIE_DECODE_ACCESSORS 1
#elif KIE_DH == 128 && KIE_MOE == 0
KIE_DECODE_ENTRY(128, 0)
#define KIE_DECODE_ACCESSORS 1
#elif KIE_DH == 128 && KIE_MOE == 1
KIE_DECODE_ENTRY(128, 1)
#elif KIE_DH == 64 && KIE_MOE == 0
KIE_DECODE_ENTRY(64, 0)
#elif KIE_DH == 64 && KIE_MOE == 1
KIE_DECODE_ENTRY(64, 1)
#else
#error "KIE_DH must be 64 or 128 and KIE_MOE 0 or 1"
#endif

#ifdef KIE_DECODE_ACCESSORS
int kernel_smem_bytes(int vec_floats, int n_desc, int n_stages, int stage_bytes) {
  return smem_total(vec_floats, n_desc, n_stages, stage_bytes);
}
int kernel_max_stages() { return kMaxStages; }
#endif

}  // namespace kie
