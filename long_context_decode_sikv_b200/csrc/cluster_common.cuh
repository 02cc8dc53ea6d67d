// Thread-block cluster primitives (sm_90+ PTX) shared by the cluster kernels:
// the CTA's rank, cluster barriers, and loads, stores and reductions on
// another CTA's shared memory (distributed shared memory).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sikv {

namespace {

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster arrives (below) and later waits;
// the wait has acquire semantics.
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }

// Arrival that publishes the whole CTA's earlier writes with one fence: the
// CTA barrier orders every thread's writes before thread 0's cluster-scope
// fence (which is cumulative), and the cluster barrier completes only after
// thread 0 arrives behind its fence, so the matching acquire wait sees them.
// The other threads arrive without fencing (a per-thread release would make
// each of them wait for its own outstanding loads and prefetches).
__device__ __forceinline__ void cluster_arrive_cta() {
    __syncthreads();
    if (threadIdx.x == 0) asm volatile("fence.acq_rel.cluster;" ::: "memory");
    asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}

// Arrival with no memory ordering: for the last barrier, which only keeps
// every CTA resident until the others are done reading its shared memory.
__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory"); }

// Address of `p` (this CTA's shared memory) in the shared memory of CTA
// `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_map(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(r)
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(rank));
    return r;
}
__device__ __forceinline__ uint32_t dsmem_ld_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ float dsmem_ld_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ float2 dsmem_ld_f2(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void dsmem_st_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void dsmem_red_add(uint32_t addr, uint32_t v) {
    asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Adds v to the word at a cluster shared-memory address; returns its old value.
__device__ __forceinline__ uint32_t dsmem_atom_add(uint32_t addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}

}  // namespace

}  // namespace sikv
