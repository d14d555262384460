// Device helpers shared by the redmoe kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace redmoe {

enum : int { DT_F32 = 0, DT_BF16 = 1, DT_INT4 = 2, DT_INT2 = 3 };

// Bits of the workspace error word.
enum : int { ERRBIT_TIMEOUT = 1, ERRBIT_STATE = 2 };

constexpr unsigned FULL = 0xffffffffu;

// Control block at the start of every workspace (256 bytes, zero between calls).
struct Control {
    unsigned bar_count;   // grid-barrier arrivals since the launch began
    unsigned bar_gen;     // blocks that have finished the launch (grid_exit)
    int err;              // ERRBIT_* set by any kernel that gave up waiting
    unsigned x_ready;     // one-row kernel: x copied from host memory into the workspace
    unsigned pad[60];
};
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

// ----------------------------------------------------------------- conversions
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

// Round-to-nearest-even fp32 -> bf16 bits (inputs are finite).
__device__ __forceinline__ uint16_t f2bf(float f) {
    uint32_t u = __float_as_uint(f);
    u += 0x7fffu + ((u >> 16) & 1u);
    return uint16_t(u >> 16);
}

// Order-preserving map of a float onto uint32 (larger float -> larger key); -0 == +0.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.0f) f = 0.0f;
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// ------------------------------------------------------------------- loads
// Streaming read-only 16-byte load: weights are read once per call, keep them out of L1.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint16_t ld_stream_u16(const void* p) {
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// L2 prefetch of the 16-byte-aligned part of [p, p + bytes): the start is rounded up
// and the end down, so the prefetched range never leaves the buffer.
__device__ __forceinline__ void prefetch_l2(const void* p, uint64_t bytes) {
    const uint64_t a = reinterpret_cast<uint64_t>(p);
    const uint64_t s = (a + 15u) & ~uint64_t(15);
    const uint64_t e = (a + bytes) & ~uint64_t(15);
    for (uint64_t q = s; q < e; q += (1u << 20)) {
        const uint32_t n = uint32_t((e - q) < (1u << 20) ? (e - q) : (1u << 20));
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(q), "r"(n) : "memory");
    }
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_relaxed_gpu(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ------------------------------------------------------- mbarrier / bulk copies
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
// Make mbarrier initialisation visible to the async proxy (bulk copies, tensor cores).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Order this thread's generic-proxy shared-memory accesses before later async-proxy ones.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Order earlier generic-proxy global writes (seen through a grid barrier) before this
// thread's later async-proxy (bulk copy) reads of global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait for the phase of `bar` with the given parity. Gives up after timeout_ns
// (or, once it has waited 20 us, as soon as another thread has recorded a timeout): sets
// ERRBIT_TIMEOUT in *err and returns false; the caller carries on with whatever the buffer
// holds. The error word is not read during the first 20 us: a global load in the polling
// loop would delay noticing a completed phase by its latency.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0u) {
            const uint64_t dt = globaltimer_ns() - t0;
            if (dt > timeout_ns || i > (1u << 26) || (dt > 20000u && ld_relaxed_gpu(err) != 0)) {
                atomicOr(err, ERRBIT_TIMEOUT);
                return false;
            }
        }
    }
}
// 1-D bulk copy global -> shared (this CTA), completion counted on `bar` in bytes.
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------------------- warp reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

// ------------------------------------------------------------ grid barrier
// Barrier across all blocks of a cooperative launch (every block is resident, so every
// block eventually arrives). Barrier number b of a launch waits until the arrival counter
// reaches (b + 1) * nblocks; arrivals are fire-and-forget reductions. Memory order comes
// from the reductions and loads themselves, with no separate fence: the block's threads
// meet at __syncthreads, then thread 0 arrives with a release (cumulative over the writes
// the barrier made it observe); a waiter polls with acquire loads and then releases its
// block (or warp) with __syncthreads (__syncwarp), which orders the block's later reads
// after the other blocks' writes. A bulk copy that reads such data still needs
// fence.proxy.async first. grid_exit() or grid_release() must end
// the launch: its last block resets the counter for the next launch. The wait is bounded:
// after `timeout_ns` (or once another block has recorded a timeout) the block records
// ERRBIT_TIMEOUT and continues, so a fault can never hang the GPU; the host reads the
// error word.
__device__ __forceinline__ void grid_barrier(Control* ctl, unsigned nblocks, unsigned index, uint64_t timeout_ns) {
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(&ctl->bar_count) : "memory");
        const unsigned target = (index + 1u) * nblocks;
        if (ld_acquire_gpu(&ctl->bar_count) < target) {
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t spins = 1; ld_acquire_gpu(&ctl->bar_count) < target; ++spins) {
                if ((spins & 63u) == 0u) {
                    const uint64_t dt = globaltimer_ns() - t0;
                    if (dt > timeout_ns || spins > (1u << 26) || (dt > 20000u && ld_relaxed_gpu(&ctl->err) != 0)) {
                        atomicOr(&ctl->err, ERRBIT_TIMEOUT);
                        break;
                    }
                }
            }
        }
    }
    __syncthreads();
}

// The two halves of grid_barrier, for work that may overlap the wait (arrive, then do
// independent work, then wait). Same bounded wait and error reporting.
__device__ __forceinline__ void grid_arrive(Control* ctl) {
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(&ctl->bar_count) : "memory");
    }
}
__device__ __forceinline__ void grid_wait(Control* ctl, unsigned nblocks, unsigned index, uint64_t timeout_ns) {
    if (threadIdx.x == 0) {
        const unsigned target = (index + 1u) * nblocks;
        if (ld_acquire_gpu(&ctl->bar_count) < target) {
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t spins = 1; ld_acquire_gpu(&ctl->bar_count) < target; ++spins) {
                if ((spins & 63u) == 0u) {
                    const uint64_t dt = globaltimer_ns() - t0;
                    if (dt > timeout_ns || spins > (1u << 26) || (dt > 20000u && ld_relaxed_gpu(&ctl->err) != 0)) {
                        atomicOr(&ctl->err, ERRBIT_TIMEOUT);
                        break;
                    }
                }
            }
        }
    }
    __syncthreads();
}

// grid_wait for the calling warp alone: lane 0 waits (same bound and error report), then
// the warp's lanes see what every block wrote before its arrive. The block's other warps
// are not held.
__device__ __forceinline__ void grid_wait_warp(Control* ctl, unsigned nblocks, unsigned index, uint64_t timeout_ns) {
    if ((threadIdx.x & 31) == 0) {
        const unsigned target = (index + 1u) * nblocks;
        if (ld_acquire_gpu(&ctl->bar_count) < target) {
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t spins = 1; ld_acquire_gpu(&ctl->bar_count) < target; ++spins) {
                if ((spins & 63u) == 0u) {
                    const uint64_t dt = globaltimer_ns() - t0;
                    if (dt > timeout_ns || spins > (1u << 26) || (dt > 20000u && ld_relaxed_gpu(&ctl->err) != 0)) {
                        atomicOr(&ctl->err, ERRBIT_TIMEOUT);
                        break;
                    }
                }
            }
        }
    }
    __syncwarp();
}

// The block has passed the launch's last wait on the barrier counters: count it out; the
// last block out resets the counters (and the x-ready flag) for the next launch. Thread 0
// calls it right after the final grid_barrier / grid_wait, so the atomic round trips of
// the reset overlap the rest of the launch instead of lengthening its tail. A launch uses
// either this or grid_exit.
__device__ __forceinline__ void grid_release(Control* ctl, unsigned nblocks) {
    if (threadIdx.x == 0) {
        const unsigned done = atomicAdd(&ctl->bar_gen, 1u);
        if (done == nblocks - 1u) {
            atomicExch(&ctl->bar_count, 0u);
            atomicExch(&ctl->bar_gen, 0u);
            atomicExch(&ctl->x_ready, 0u);
        }
    }
}

// End of a launch that used grid_barrier: the last block out resets the counters.
__device__ __forceinline__ void grid_exit(Control* ctl, unsigned nblocks) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned done = atomicAdd(&ctl->bar_gen, 1u);
        if (done == nblocks - 1u) {
            atomicExch(&ctl->bar_count, 0u);
            atomicExch(&ctl->bar_gen, 0u);
        }
    }
}

}  // namespace redmoe
