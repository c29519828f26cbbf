// Shared helpers of the moefp8 CUDA library (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moefp8.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "moefp8 kernels target sm_100a (B200) only"
#endif

namespace moe {

// ------------------------------------------------------------------ host
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int check_launch() {
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Number of SMs of the current device (cached per device).
int sm_count();

// Validates a MoE shape; returns MOE_OK or an error code.
int validate_shape(const MoeShape* s);

// True when the current device is an sm_100 part.
bool device_is_sm100();

// --------------------------------------------------------------- device
__device__ __forceinline__ void set_status(int* st, int code) {
    if (st) atomicCAS(st, 0, code);
}

// Two fp32 values -> two E4M3 codes, nearest-even, saturating to +-448.
// Byte 0 of the result holds `lo`, byte 1 holds `hi`.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Online scale rule of the library: scale = fp32(amax/448), inverse =
// fp32(448/amax); amax == 0 -> scale 1, inverse 1 (codes keep the sign of 0).
__device__ __forceinline__ void scale_from_amax(float amax, float& scale, float& inv) {
    if (amax == 0.0f) {
        scale = 1.0f;
        inv = 1.0f;
    } else {
        scale = __fdiv_rn(amax, 448.0f);
        inv = __fdiv_rn(448.0f, amax);
    }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// A wait that has not finished after this many nanoseconds is abandoned and
// reported as MOE_DEV_TIMEOUT.  Real waits in these kernels last microseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

}  // namespace moe
