// Global stores with an L2 evict-first policy.
//
// The quantisers write sketches and codes that are read again only by a
// later call. Stored with the evict-first policy, those lines are the first
// the L2 gives up while the quantiser still streams its input, so the
// write-back of the quantiser's own output happens during the quantiser
// instead of being left, dirty, in L2 for the next kernel to evict. The
// stores skip L1 too: nothing in the writing kernel reads them back.
#pragma once

#include <stdint.h>

namespace qjl_hint {

__device__ __forceinline__ uint64_t evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void st_u32(uint32_t* p, uint32_t v, uint64_t pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.b32 [%0], %1, %2;" ::"l"(p), "r"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_u16(uint16_t* p, uint16_t v, uint64_t pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(p), "h"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_f32(float* p, float v, uint64_t pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_v2(uint32_t* p, uint32_t a, uint32_t b, uint64_t pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v2.b32 [%0], {%1, %2}, %3;" ::"l"(p), "r"(a), "r"(b),
               "l"(pol)
               : "memory");
}

__device__ __forceinline__ void st_v4(uint32_t* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint64_t pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(a),
               "r"(b), "r"(c), "r"(d), "l"(pol)
               : "memory");
}

}  // namespace qjl_hint
