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

// False when p is memory the GPU cannot address (pageable host memory that
// was never registered with CUDA); device, managed and pinned host memory
// pass.  NULL passes (callers check required pointers separately).
bool device_accessible(const void* p);

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

// Power-of-two scale option (UE8M0 scale bytes, for the block-scaled MMA
// form): e = the smallest integer with amax <= 448 * 2^e, clamped to
// [-127, 127], 0 for amax = 0; the scale is 2^e (byte e + 127) and the code
// of v is E4M3(v * 2^-e).  Every comparison is exact in FP64.
__device__ __forceinline__ int pow2_exponent(float amax) {
    if (!(amax > 0.0f)) return 0;
    const double a = (double)amax;
    int e = int((__double_as_longlong(a) >> 52) & 0x7FF) - 1023 - 9;  // too small
    // 448 * 2^e = 1.75 * 2^(e + 8), built from its bits
    while (a > __longlong_as_double((int64_t(e + 8 + 1023) << 52) | (int64_t(3) << 50))) ++e;
    return max(-127, min(127, e));
}
// 2^-e as fp32 for e in [-127, 127] (2^-127 is the subnormal 0x00400000)
__device__ __forceinline__ float pow2_inverse(int e) {
    return e < 127 ? __int_as_float((127 - e) << 23) : __int_as_float(0x00400000);
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
// The limit is a kernel argument: wait_limit_ns() gives it, this default
// unless MOEFP8_WAIT_LIMIT_NS is set in the environment.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Bounded wait limit of the next launch (host; read at every call).
uint64_t wait_limit_ns();

// Host-driven fault injection (MOEFP8_FAULT in the environment, read at
// every call): kFaultGemmProducer makes the single-CTA grouped GEMM's TMA
// producer withhold the loads of its first stage, so that the MMA issuer's
// bounded wait on that stage runs out (MOE_DEV_TIMEOUT) and the kernel
// unwinds.  Nothing faults, traps or hangs: the wait limit ends it.
enum FaultKind { kFaultNone = 0, kFaultGemmProducer = 1 };
int fault_injection();

}  // namespace moe
