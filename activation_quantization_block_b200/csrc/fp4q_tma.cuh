// TMA tile pipeline for the fp4q streaming kernels (sm_100a).
//
// A bf16 matrix is read as 2-D tiles of 128 rows x 64 elements (128 bytes per
// row, 16 KB per tile) by cp.async.bulk.tensor into shared memory with the
// 128-byte swizzle: the 16-byte chunk c of tile row r lands at chunk c ^ (r & 7).
// A thread that owns the 64-byte unit (row r, half h) reads its four chunks
// 4h..4h+3 at (4h + j) ^ (r & 7); in every phase of eight lanes the eight
// requests hit eight different 16-byte bank groups, so the reads are
// conflict-free without any register permutation.
//
// Each CTA runs a ring of kStages tiles guarded by one mbarrier each: thread 0
// arms the barrier with the tile's byte count and issues the copy; all threads
// wait on the barrier's phase, consume the tile, meet at __syncthreads, and
// thread 0 refills the slot with the tile kStages ahead.  No multicast and no
// clusters: every CTA fetches its own tiles from this GPU's memory.
//
// Every wait is bounded (kWaitLimitNs of the global timer).  A CTA whose wait
// runs out records kErrPipelineTimeout in the device error word, waits (again
// bounded) for the copies it has in flight, and returns.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace fp4q {

constexpr int kTileRows = 128;                 // tile rows (64 bf16 = 128 bytes each)
constexpr int kTileCols = 64;                  // elements per tile row
constexpr int kTileBytes = kTileRows * 128;    // 16 KB
constexpr int kStages = 4;                     // tiles in flight per CTA
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Bits of the device error word.
constexpr unsigned kErrPipelineTimeout = 1u;
constexpr unsigned kErrOutOfBounds = 2u;

#ifndef FP4Q_DEBUG
#define FP4Q_DEBUG 0
#endif

// Bounds check of a global access of `len` bytes at byte offset `off` into a
// buffer of `extent` bytes, done only in builds with FP4Q_DEBUG (otherwise
// always true, and compiled away).  An access outside the buffer sets
// kErrOutOfBounds in the error words `err`; the first such access also leaves
// its site (a number naming the access) and its offset; the caller skips it.
__device__ __forceinline__ bool in_bounds(int64_t off, int64_t len, int64_t extent, unsigned site, unsigned* err)
{
    if (!FP4Q_DEBUG) return true;
    if (off >= 0 && len >= 0 && off <= extent - len) return true;
    atomicOr(err, kErrOutOfBounds);
    if (atomicCAS(err + 1, 0u, site) == 0u) {
        atomicExch(err + 2, (unsigned)((uint64_t)off & 0xFFFFFFFFu));
        atomicExch(err + 3, (unsigned)((uint64_t)off >> 32));
    }
    return false;
}

// Sites of the checked accesses (fp4q_device_error_site).
enum : unsigned {
    kSiteCodesStore = 1, kSiteScalesStore, kSiteAmaxPartialStore, kSiteSsePartialStore, kSiteAmaxPartialLoad,
    kSiteSsePartialLoad, kSiteCodesLoad, kSiteScalesLoad, kSiteScalarStore, kSiteScalarLoad, kSiteOutlierRowLoad,
    kSiteBulkStore, kSiteSlotStore, kSiteCountStore, kSiteScatterStore, kSitePlanesStore, kSiteSfStore,
    kSiteGemmStore, kSiteCountLoad, kSiteSlotLoad
};

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arm(uint32_t bar, uint32_t tx_bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(tx_bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// 2-D tiled load of box {64, 128} at element coordinates (x, y) into shared memory.
__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// 2-D tiled store of a shared-memory tile to (x, y); out-of-range parts are clipped.
__device__ __forceinline__ void tma_store_tile(const CUtensorMap* map, int x, int y, uint32_t src)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                 ::"l"(map), "r"(x), "r"(y), "r"(src)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until the shared-memory sources of all committed bulk stores have been read.
__device__ __forceinline__ void bulk_wait_reads() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Wait until the sources of all but the most recent committed bulk store have been read.
__device__ __forceinline__ void bulk_wait_reads_but_last() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }

// Wait until all committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Make generic-proxy shared-memory writes visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Programmatic dependent launch: wait for the preceding kernel's results /
// allow the following kernel to start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Byte address of 16-byte chunk c of tile row r in a swizzled tile.
__device__ __forceinline__ uint32_t tile_chunk(uint32_t tile, uint32_t r, uint32_t c)
{
    return tile + r * 128u + ((c ^ (r & 7u)) << 4);
}

}  // namespace fp4q
