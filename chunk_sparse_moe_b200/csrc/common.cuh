// common.cuh -- shared definitions of the BlockFFN CUDA library: workspace
// control block, device-side error recording and bounded waits.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace bffn {

// Status codes, identical to blockffn_status in include/blockffn.h.
enum : int32_t {
    kOk = 0,
    kErrInvalidArg = 1,
    kErrUnsupported = 2,
    kErrCuda = 3,
    kErrTimeout = 4,
    kErrWorkspace = 5,
};

// Which wait ran out (the "detail" of a timeout).
enum : int32_t {
    kWaitEmpty = 1,      // producer waiting for a free pipeline stage
    kWaitFullW = 2,      // MMA waiting for a weight/activation tile
    kWaitFullH = 3,      // MMA waiting for a gated-activation tile
    kWaitAccFull = 4,    // epilogue waiting for an accumulator
    kWaitAccEmpty = 5,   // MMA waiting for a free accumulator
    kWaitFlag = 6,       // activation loader waiting for another block's result
    kWaitDrain = 7,      // teardown waiting for its own copies in flight
    kWaitMmaDone = 8,    // teardown waiting for the last MMAs
    kWaitPeers = 9,      // a split unit's block waiting for the other contributors
};

// Control block at offset 0 of every forward workspace (256 bytes reserved).
struct Ctl {
    int32_t status;        // first device-side error (sticky until reset)
    int32_t detail;        // which wait / check
    uint32_t epoch;        // number of completed forward launches (flag stamp)
    uint32_t done;         // thread blocks of the current launch that finished
    uint32_t issued[2];    // by launch parity: blocks that issued their last expert-in load
    uint32_t pad[58];
};
static_assert(sizeof(Ctl) == 256, "control block is 256 bytes");

__device__ __forceinline__ void record_error(Ctl* ctl, int32_t code, int32_t detail) {
    if (atomicCAS(&ctl->status, 0, code) == 0) atomicExch(&ctl->detail, detail);
}

// Spin on an mbarrier phase for at most limit_ns.  Gives up early when another
// role of the block has aborted.  On running out, records a timeout and sets
// the block's abort flag.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                         volatile int* abort, Ctl* ctl, int32_t detail) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_error(ctl, kErrTimeout, detail);
            *abort = 1;
            return false;
        }
    }
}

// The same wait made by all 32 lanes of a warp together, with one outcome for
// the whole warp (lane 0's observations decide), so the warp's control flow stays
// uniform: a role whose loop runs on every lane and issues through one elected
// lane keeps its instructions flowing at the converged rate, where a loop run by
// one lane alone while the others wait was measured to issue tcgen05 work at
// about half that rate.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                              volatile int* abort, Ctl* ctl, int32_t detail) {
    if (__shfl_sync(0xffffffffu, mbar_try_wait(bar, parity) ? 1 : 0, 0)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        int st = mbar_try_wait(bar, parity) ? 1 : (*abort ? 2 : (globaltimer_ns() - t0 > limit_ns ? 3 : 0));
        st = __shfl_sync(0xffffffffu, st, 0);
        if (st == 1) return true;
        if (st == 2) return false;
        if (st == 3) {
            if ((threadIdx.x & 31) == 0) {
                record_error(ctl, kErrTimeout, detail);
                *abort = 1;
            }
            __syncwarp();
            return false;
        }
    }
}

// Same, acquiring at cluster scope (for barriers that blocks of the cluster
// arrive on remotely).
__device__ __forceinline__ bool wait_bar_cluster(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                 volatile int* abort, Ctl* ctl, int32_t detail) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_error(ctl, kErrTimeout, detail);
            *abort = 1;
            return false;
        }
    }
}

// Same, without the abort short-cut: used at teardown to let copies land.
__device__ __forceinline__ bool wait_bar_drain(uint64_t* bar, uint32_t parity,
                                               uint64_t limit_ns, Ctl* ctl) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_error(ctl, kErrTimeout, kWaitDrain);
            return false;
        }
    }
}

// Spin until the counter reaches want (acquire), bounded.  detail tells which
// wait this is when it runs out.
__device__ __forceinline__ bool wait_count(const uint32_t* ctr, uint32_t want, uint64_t limit_ns,
                                           volatile int* abort, Ctl* ctl,
                                           int32_t detail = kWaitFlag) {
    if (ld_acquire_gpu(ctr) >= want) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(32);
        if (ld_acquire_gpu(ctr) >= want) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_error(ctl, kErrTimeout, detail);
            *abort = 1;
            return false;
        }
    }
}

// Named barrier over nthreads threads (whole warps).  The warp first gathers
// all its lanes, so the aligned barrier is executed by a converged warp even
// right after a branch that only one lane took (for instance lane 0 in a
// bounded wait while lanes 1-31 went ahead).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    __syncwarp();
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__host__ __device__ inline long long ceil_div_ll(long long a, long long b) {
    return (a + b - 1) / b;
}

}  // namespace bffn
