// tcgen05 / TMA glue shared by kernels outside the grouped GEMM (sm_100a).
// Shared-memory operand tiles are K-major with 128-byte rows and the
// 128-byte swizzle (8-row atoms, 1024 bytes apart); every wait is bounded.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {

// 2D uint8 tensor map over [rows, cols] (cols contiguous), box = [box_rows,
// 128 bytes], 128-byte swizzle (defined with the grouped GEMM).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "n"(20000)
        : "memory");
    return ok != 0;
}

// Waits for the phase with `parity`; gives up (raising *abort and the
// device status) after limit_ns, or when *abort is already raised.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* abort,
                                          int* dev_status, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0) {
            if (*reinterpret_cast<volatile int*>(abort)) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                atomicExch(abort, 1);
                set_status(dev_status, MOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
}

// Waits for work already in flight (TMA copies, MMAs) before a CTA frees
// what that work writes: like mbar_wait but it does not stop when the CTA
// has aborted; it still gives up after limit_ns.
__device__ __forceinline__ bool mbar_quiesce(uint32_t bar, uint32_t parity, int* dev_status,
                                             uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0 && globaltimer_ns() - t0 > limit_ns) {
            set_status(dev_status, MOE_DEV_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory descriptor of a K-major tile with 128-byte rows, 128-byte
// swizzle, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= uint64_t((saddr & 0x3FFFFu) >> 4);  // start address
    d |= uint64_t(16 >> 4) << 16;            // leading byte offset (unused here)
    d |= uint64_t(1024 >> 4) << 32;          // stride byte offset: 8 rows x 128 B
    d |= uint64_t(1) << 46;                  // descriptor version for tcgen05
    d |= uint64_t(2) << 61;                  // 128-byte swizzle
    return d;
}

// kind::i8 instruction descriptor: D s32, A and B signed 8-bit, both K-major.
__device__ __forceinline__ uint32_t idesc_s8(int m, int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) |
           (uint32_t(m >> 4) << 24);
}

__device__ __forceinline__ void mma_s8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 16 consecutive TMEM columns of this warp's 32 lanes -> 16 registers; the
// wait for the load is part of the same statement.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

}  // namespace tc
}  // namespace moe
