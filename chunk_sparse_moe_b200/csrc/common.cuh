// common.cuh -- shared definitions of the BlockFFN CUDA library: workspace
// control block, device-side error recording and bounded waits.
#pragma once
#include <cstddef>
#include <cstdint>
#include <initializer_list>
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
    kShapeKey = 10,      // (workspace error) bound to other shapes or another gating mode
    kUnionTables = 11,   // (invalid argument) caller's counts / idx disagree with its token masks
};

// Control block at offset 0 of every forward workspace (256 bytes reserved).
struct Ctl {
    int32_t status;        // first device-side error (sticky until reset)
    int32_t detail;        // which wait / check
    uint32_t plan_done;    // blocks of the current group-plan launch that finished (the last resets it)
    uint32_t unused_;
    uint32_t issued[2];    // by launch parity: blocks that issued their last expert-in load
    // The shapes, dtype, gating mode and kernel the workspace's layout was made
    // for, claimed by the first launch after a reset (0 = not yet bound).  A
    // launch whose key differs records kErrWorkspace and computes nothing: its
    // counters and tables would sit at other offsets.
    unsigned long long shape_key;
    // One ticket per thread block of every launch on this workspace: block b of
    // launch k draws a ticket in [k*G, (k+1)*G) (G = the launch's grid, fixed for
    // a workspace by its shape key), so ticket / G is the launch's index with one
    // atomic and no end-of-launch bookkeeping.  64 bits: it never wraps.
    unsigned long long ticket;
    uint32_t pad[54];
};
static_assert(sizeof(Ctl) == 256, "control block is 256 bytes");

__device__ __forceinline__ void record_error(Ctl* ctl, int32_t code, int32_t detail) {
    if (atomicCAS(&ctl->status, 0, code) == 0) atomicExch(&ctl->detail, detail);
}

// Host-side key of a launch's workspace layout: FNV-1a over the values that
// decide it.  Never 0 (0 marks an unbound workspace).
inline unsigned long long shape_key(std::initializer_list<long long> vals) {
    unsigned long long h = 1469598103934665603ull;
    for (long long v : vals) {
        for (int b = 0; b < 8; ++b) {
            h ^= (unsigned long long)((v >> (8 * b)) & 0xff);
            h *= 1099511628211ull;
        }
    }
    return h | 1ull;
}

// Claim the workspace for this launch's key, or find it bound to the same key.
// Returns the previous key; the caller compares (one atomic, issued beside the
// prologue's other control-block accesses so its latency overlaps theirs).
__device__ __forceinline__ unsigned long long claim_shape_key(Ctl* ctl, unsigned long long key) {
    return atomicCAS(&ctl->shape_key, 0ull, key);
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
