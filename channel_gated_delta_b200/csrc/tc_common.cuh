// tcgen05 / TMEM / mbarrier helpers for sm_100a (inline PTX).
//
// Shared-memory operand tiles use one physical layout, "row tiles": a tile of
// R rows whose 16-bit columns are grouped in blocks of 64 (128 bytes per
// row); block b starts at b * R * 128 bytes, row r of a block at r * 128, and
// the 16-byte chunk c of a row is stored at chunk position (c ^ (r & 7)) --
// the 128-byte swizzle.  Every tile base is 1024-byte aligned.
//
// One row tile can feed the tensor core in two ways:
//  * K-major: rows are the M (or N) index, columns the contraction index K;
//  * MN-major: rows are the contraction index K, columns the M (or N) index.
// The descriptors below encode both (tcgen05 shared-memory matrix
// descriptor, version 1, 128-byte swizzle; see the layout notes of CUTLASS
// cute/atom/mma_traits_sm100.hpp for the canonical forms).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace gdelta {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of 16-bit element (r, col) in a row tile of R rows.
__device__ __forceinline__ uint32_t tile_off(int R, int r, int col) {
    const int b = col >> 6, c = (col & 63) >> 3, e = col & 7;
    return (uint32_t)(b * R * 128 + r * 128 + ((c ^ (r & 7)) << 4) + e * 2);
}
// Byte offset of the 16-byte chunk holding columns [8*c8, 8*c8+8) of row r.
__device__ __forceinline__ uint32_t tile_chunk_off(int R, int r, int c8) {
    const int b = c8 >> 3, c = c8 & 7;
    return (uint32_t)(b * R * 128 + r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for sm_100
    d |= (uint64_t)2 << 61;   // 128-byte swizzle
    return d;
}

// K-major view: rows [row0, row0 + M) of a tile with R rows; K-step ks covers
// columns [16 ks, 16 ks + 16).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int R, int row0, int ks) {
    const int col = ks * 16;
    const uint32_t a = tile + (uint32_t)((col >> 6) * R * 128 + row0 * 128 + (col & 63) * 2);
    return make_desc(a, 16, 1024);
}

// MN-major view: K-step ks covers rows [row0 + 16 ks, row0 + 16 ks + 16);
// the M/N index runs along the columns (blocks of 64 at stride R*128).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int R, int row0, int ks) {
    const uint32_t a = tile + (uint32_t)((row0 + ks * 16) * 128);
    return make_desc(a, (uint32_t)R * 128u, 1024);
}

// The descriptor of K-step ks from that of step 0: only the start-address field
// (address >> 4, bits 0-13) moves, and shared-memory addresses stay below 2^18,
// so a plain add never carries out of the field.  With ks a compile-time
// constant this is one 64-bit add per MMA instead of rebuilding the descriptor
// (in a one-CTA test that rebuilt descriptors with run-time layout choices, one
// issuing thread managed an MMA per 100 cycles, against 72 with ready ones).
__device__ __forceinline__ uint64_t desc_kmajor_step(uint64_t d0, int R, int ks) {
    return d0 + (uint64_t)((ks >> 2) * R * 8 + (ks & 3) * 2);
}
__device__ __forceinline__ uint64_t desc_mnmajor_step(uint64_t d0, int ks) { return d0 + (uint64_t)(ks * 128); }

// Instruction descriptor, kind::f16 with fp16 A and B, fp32 accumulator.
__device__ __forceinline__ uint32_t idesc_f16(int M, int N, bool a_mn, bool b_mn, bool a_neg) {
    uint32_t d = 0;
    d |= 1u << 4;                              // D format: f32
    // A, B format: f16 (0) at bits 7..9 and 10..12
    d |= (a_neg ? 1u : 0u) << 13;
    d |= (a_mn ? 1u : 0u) << 15;
    d |= (b_mn ? 1u : 0u) << 16;
    d |= (uint32_t)(N >> 3) << 17;
    d |= (uint32_t)(M >> 4) << 24;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 A and B (format code 1 in both
// operand fields), fp32 accumulator.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    uint32_t d = 0;
    d |= 1u << 4;                              // D format: f32
    d |= 1u << 7;                              // A format: bf16
    d |= 1u << 10;                             // B format: bf16
    d |= (a_mn ? 1u : 0u) << 15;
    d |= (b_mn ? 1u : 0u) << 16;
    d |= (uint32_t)(N >> 3) << 17;
    d |= (uint32_t)(M >> 4) << 24;
    return d;
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, bool accumulate) {
    const uint32_t acc = accumulate ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc));
}

// Arrives once on the mbarrier when all previously issued MMAs of this thread complete.
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Generic-proxy shared-memory writes -> visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMEM allocation (one warp, .sync.aligned).  The allocated base address is
// written to *dst_smem.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (32 * (warp % 4) + i) of the address's lane base, columns col..col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Two 32-column loads issued back to back, one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t tb, float (&va)[32], float (&vb)[32]) {
    uint32_t r[64];
#define GD_LD32(base, addr)                                                                                     \
    asm volatile(                                                                                               \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                                               \
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"                                               \
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                              \
        : "=r"(r[base + 0]), "=r"(r[base + 1]), "=r"(r[base + 2]), "=r"(r[base + 3]), "=r"(r[base + 4]),        \
          "=r"(r[base + 5]), "=r"(r[base + 6]), "=r"(r[base + 7]), "=r"(r[base + 8]), "=r"(r[base + 9]),        \
          "=r"(r[base + 10]), "=r"(r[base + 11]), "=r"(r[base + 12]), "=r"(r[base + 13]), "=r"(r[base + 14]),   \
          "=r"(r[base + 15]), "=r"(r[base + 16]), "=r"(r[base + 17]), "=r"(r[base + 18]), "=r"(r[base + 19]),   \
          "=r"(r[base + 20]), "=r"(r[base + 21]), "=r"(r[base + 22]), "=r"(r[base + 23]), "=r"(r[base + 24]),   \
          "=r"(r[base + 25]), "=r"(r[base + 26]), "=r"(r[base + 27]), "=r"(r[base + 28]), "=r"(r[base + 29]),   \
          "=r"(r[base + 30]), "=r"(r[base + 31])                                                                \
        : "r"(addr))
    GD_LD32(0, ta);
    GD_LD32(32, tb);
#undef GD_LD32
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        va[i] = __uint_as_float(r[i]);
        vb[i] = __uint_as_float(r[32 + i]);
    }
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- programmatic dependent launch ----
// The next kernel in the stream, when launched with launch_dependent, may start
// once every CTA of this grid has executed this (or exited).
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Wait until the grid this one depends on has completed and its memory
// operations are visible (returns at once when there is none).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---- mbarriers (shared::cta) ----
__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t mbar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(mbar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after `limit` polls and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, uint32_t limit = (1u << 20)) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(mbar, parity)) return true;
    return false;
}

// One arrival on a local mbarrier (release at CTA scope).
__device__ __forceinline__ void mbar_arrive_local(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

// One arrival on a local mbarrier without release semantics: it does not wait
// for this thread's earlier global stores to be performed.  For handing back
// a TMEM region whose reads completed (tcgen05.wait::ld) before the arrival.
__device__ __forceinline__ void mbar_arrive_local_relaxed(uint32_t mbar) {
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

// One expected arrival that also announces `bytes` of asynchronous transfers.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}

// Bulk copy of `bytes` contiguous bytes global -> this CTA's shared memory
// (both addresses 16-byte aligned, size a multiple of 16); completion is
// counted on the mbarrier's transaction count.  No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst_smem, const void *src, uint32_t bytes, uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst_smem),
        "l"(src), "r"(bytes), "r"(mbar)
        : "memory");
}

// Bulk copy shared -> global (bulk-group completion); see bulk_commit / bulk_wait_read.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src_smem), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared-memory sources of all committed bulk stores may be reused.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until all committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 2-D tiled TMA load of one box of the tensor map at `tmap` (a kernel parameter
// in param space, passed by generic address) into this CTA's shared memory,
// completion counted on the mbarrier.  x is the innermost coordinate (it must
// be a multiple of 16 bytes' worth of elements); no multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst_smem, const void *tmap, int x, int y, uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst_smem),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}

// 4-D tiled TMA load (coordinates innermost first); otherwise as tma_load_2d.
__device__ __forceinline__ void tma_load_4d(uint32_t dst_smem, const void *tmap, int x, int y, int z, int w,
                                            uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(dst_smem),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(mbar)
        : "memory");
}

// 2-D tiled TMA store of one box from this CTA's shared memory to the tensor
// map's global memory (bulk-group completion: bulk_commit, then
// bulk_wait_read_n / bulk_wait_all).  x, y are the box's first column and row,
// both non-negative, x a multiple of 16 bytes' worth of elements; rows and
// columns beyond the tensor's extent are not written.  The sources must be made
// visible to the async proxy first (fence_proxy_async by the writing threads).
__device__ __forceinline__ void tma_store_2d(const void *tmap, uint32_t src_smem, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(src_smem), "r"(x), "r"(y)
                 : "memory");
}
// Wait until at most N committed bulk-store groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read_n() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Hint: bring `bytes` (a multiple of 16) of global memory into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---- thread-block clusters: rank, peer shared-memory addresses, barriers ----
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t caddr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(caddr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t caddr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(caddr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_s32(uint32_t caddr, int v) {
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(caddr), "r"(v) : "memory");
}
// 4-byte store into another CTA's shared memory whose completion is counted
// on that CTA's mbarrier (transaction bytes); it orders nothing else, so it
// does not wait for this thread's earlier global stores.
__device__ __forceinline__ void st_async_f32(uint32_t caddr, float v, uint32_t cbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(caddr),
                 "r"(__float_as_uint(v)), "r"(cbar)
                 : "memory");
}
__device__ __forceinline__ void st_async_s32(uint32_t caddr, int v, uint32_t cbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(caddr), "r"(v),
                 "r"(cbar)
                 : "memory");
}

// One arrival on an mbarrier of another CTA of the cluster, releasing this
// thread's prior writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
// Bounded wait on a local mbarrier completed from another CTA of the cluster.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t mbar, uint32_t parity, uint32_t limit = (1u << 20)) {
    for (uint32_t i = 0; i < limit; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}
// All threads of all CTAs of the cluster.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 32-byte global accesses (sm_100): one full sector per thread and instruction;
// the address must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void *p, const uint4 &a, const uint4 &b) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
                 "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}
__device__ __forceinline__ void ld_global_nc_v8(const void *p, uint4 &a, uint4 &b) {
    asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Host: launch `kernel` as a programmatic dependent of the kernel before it in
// `stream` (cudaLaunchAttributeProgrammaticStreamSerialization): its CTAs may
// start once every CTA of that kernel has executed grid_launch_dependents, and
// it must call grid_dependency_wait before reading what that kernel writes.
// Cluster dimensions come from the kernel's own attribute.  A runtime that
// refuses the attribute gets an ordinary launch (then the wait returns at once).
template <typename... Params, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) {
        (void)cudaGetLastError();                 // clear the refusal, then launch in order
        cfg.numAttrs = 0;
        e = cudaLaunchKernelEx(&cfg, kernel, args...);
    }
    return e;
}

}  // namespace tc
}  // namespace gdelta
