// common.cuh -- helpers shared by the libmoedispatch kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "moedispatch.h"

namespace md {

// ---------------------------------------------------------------- host side

// Host-side count of enqueued kernels / memsets (md_launch_count).
void count_launches(int n);   // kernels enqueued
void count_memsets(int n);    // device memsets and device-to-device copies enqueued

// Test hooks (md_set_test_hooks); the defaults leave every kernel unchanged.
long long hook_poll_limit(long long dflt);
int hook_layout_skip_tile();        // -1: none
long long hook_expand_skip_unit();  // -1: none

// Kernel choice of md_dispatch_permute (md_set_permute_path) and launch form
// of md_dispatch_layout (md_set_layout_path).
int permute_path();
int layout_path();

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Report a failed launch; clears the error so later calls are not blamed.
inline int launch_status()
{
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MD_OK : MD_ERR_CUDA;
}

inline int clear_status(int32_t *dev_status, cudaStream_t s)
{
    if (!dev_status) return MD_OK;
    count_memsets(1);
    return cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) == cudaSuccess ? MD_OK : MD_ERR_CUDA;
}

// SMs of the current device (cached per device)
inline int sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    cudaGetDevice(&dev);
    int n = cache[dev & 63].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cache[dev & 63].store(n, std::memory_order_relaxed);
    }
    return n;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Run f() once per device of the process (function attributes are per device).
template <class F>
inline void once_per_device(std::atomic<uint64_t> &done, F f)
{
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return;
    f();
    done.fetch_or(bit, std::memory_order_acq_rel);
}

// -------------------------------------------------------------- device side

// Record a data error; the first error code written wins.
__device__ __forceinline__ void report(int32_t *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// 16-byte streaming load (read once) and store (written once).
__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(uint4 *p, uint4 v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// bf16 pair in a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Two floats -> bf16 pair, round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ------------------------------------------- TMA bulk copies and mbarriers
// Untiled bulk copies (cp.async.bulk): both addresses 16-byte aligned, the
// size a multiple of 16.  A load into shared memory completes on an mbarrier
// (transaction bytes); stores from shared memory are tracked per thread in
// bulk groups.

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// make barrier initialisation visible to the async (bulk copy) proxy
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// plain arrive (no transaction bytes): completes a phase that has no copy
__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}

// Wait for phase `parity` of `bar` with a bounded number of polls; false if
// the bound ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, long long polls)
{
    for (long long n = 0; n < polls; ++n)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src, uint32_t bytes,
                                          uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_store(void *dst, const void *src_smem, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_addr(src_smem)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// at most N of this thread's bulk groups may still be reading shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// all of this thread's bulk groups complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

}  // namespace md
