// Shared device-side pieces of libbsa: the problem geometry (block slot -> raster token),
// the device error word, bounded mbarrier waits and thin inline-PTX wrappers for the
// sm_100a instructions the kernels use (cp.async, mbarrier, tcgen05).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/bsa.h"

namespace bsa {

// ------------------------------------------------------------------------ geometry

// Everything a kernel needs to map a block slot to a raster token.
struct Geom {
    int heads, N, d, B;
    int T, H, W, text;
    int tt, th, tw;       // tile shape
    int nb, nbv, nbt;     // blocks: total, video, text
    int Nv;               // video tokens
    int slab;             // tokens per full tile slab along t: tt*H*W
};

// Raster token index held by block slot `s` (0 <= s < nb*B), or -1 for a padding slot.
// Tiles are visited in raster order of tile coordinates and truncated at the grid edge;
// tokens inside a tile are in raster order; blocks cut that concatenation every B tokens.
__host__ __device__ inline int slot_to_token(const Geom& g, int s) {
    const int video_slots = g.nbv * g.B;
    if (s >= video_slots) {
        const int t = s - video_slots;
        return t < g.text ? g.Nv + t : -1;
    }
    if (s >= g.Nv) return -1;
    const int a = s / g.slab;                              // tile slab along t
    int r = s - a * g.slab;
    const int ta = min(g.tt, g.T - a * g.tt);              // frames in this slab
    const int row_tokens = ta * g.th * g.W;                 // tokens per full tile row
    const int b = r / row_tokens;
    r -= b * row_tokens;
    const int hb = min(g.th, g.H - b * g.th);              // rows in this tile row
    const int col_tokens = ta * hb * g.tw;                  // tokens per full tile
    const int c = r / col_tokens;
    r -= c * col_tokens;
    const int wc = min(g.tw, g.W - c * g.tw);              // columns in this tile
    const int lt = r / (hb * wc);
    const int rem = r - lt * hb * wc;
    const int ly = rem / wc;
    const int lx = rem - ly * wc;
    return ((a * g.tt + lt) * g.H + (b * g.th + ly)) * g.W + (c * g.tw + lx);
}

// Block-slot table: perm[s] = raster token of block slot s (-1 = padding), s < nb*B.
// Built once per call, so kernels look tokens up instead of dividing per row.
__global__ void perm_kernel(Geom g, int* perm) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s < g.nb * g.B) perm[s] = slot_to_token(g, s);
}

// Number of real tokens in block i.
__host__ __device__ inline int block_count(const Geom& g, int i) {
    if (i < g.nbv) return min(g.B, g.Nv - i * g.B);
    return min(g.B, g.text - (i - g.nbv) * g.B);
}

// ------------------------------------------------------------------- error word

// Device error word of this library (one per device): 0 = ok, else the BSA_ERR_* code of the
// first device-side problem. Sticky: it keeps that first code until bsa_device_status reads
// and clears it. No kernel reads it, so a word left set by an earlier call changes nothing
// in later calls.
__device__ int g_error_word;

// Number of bounded waits that ran out on this device, ever. A kernel reads it once at entry;
// its waits give up early when it has moved since (another wait of the same launch, or of a
// launch running beside it, ran out), so the roles of a CTA wind down together instead of
// each waiting out its own limit. Errors other than a timeout do not move it.
__device__ unsigned int g_timeouts;

__device__ inline void raise_error(int code) { atomicCAS(&g_error_word, 0, code); }
__device__ inline void raise_timeout() {
    raise_error(BSA_ERR_TIMEOUT);
    atomicAdd(&g_timeouts, 1u);
}
__device__ inline unsigned timeout_epoch() { return *(volatile unsigned*)&g_timeouts; }
__device__ inline bool timed_out_since(unsigned epoch) { return *(volatile unsigned*)&g_timeouts != epoch; }

// About 2 s at the highest SM clock: any wait longer than this is treated as a hang.
#ifndef BSA_WAIT_LIMIT_CYCLES
#define BSA_WAIT_LIMIT_CYCLES 4000000000LL
#endif
constexpr long long kWaitLimitCycles = BSA_WAIT_LIMIT_CYCLES;

// --------------------------------------------------------------------- PTX: misc

__device__ inline uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline uint32_t elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(pred));
    return pred;
}

// ------------------------------------------------------------------ PTX: mbarrier

__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ inline void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ inline void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}"
                 ::"r"(smem_u32(bar)) : "memory");
}

// Suspends the thread (no spinning) until the phase with the given parity completes or the
// hinted time (in ns) passes; returns whether it completed.
__device__ inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u) : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete. Gives up (returning false) after
// kWaitLimitCycles, raising BSA_ERR_TIMEOUT, or as soon as a wait elsewhere has run out since
// the kernel read `epoch` (timeout_epoch() at entry).
__device__ inline bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned epoch) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (timed_out_since(epoch)) return false;
        if (clock64() - t0 > kWaitLimitCycles) { raise_timeout(); return false; }
    }
    return true;
}

// Teardown wait: for work already issued to the hardware (tensor-core operations, copies),
// which completes whatever else went wrong. Stops only at the cycle limit.
__device__ inline bool mbar_drain(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) { raise_timeout(); return false; }
    }
    return true;
}

// 16-byte shared-memory accesses by address.
__device__ inline void st_shared_v4(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}
__device__ inline uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// ----------------------------------------------------------- PTX: thread-block clusters

__device__ inline uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address in CTA `rank`'s shared memory of the object at `addr` in this CTA's (same offset).
__device__ inline uint32_t cluster_map(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Asynchronous 8-byte store into another CTA's shared memory; on arrival it counts its bytes
// against that CTA's mbarrier `cluster_bar` (complete_tx). The issuing thread does not wait.
__device__ inline void st_async_f32x2(uint32_t cluster_addr, float a, float b, uint32_t cluster_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];"
                 ::"r"(cluster_addr), "f"(a), "f"(b), "r"(cluster_bar) : "memory");
}

// Arrive on a local mbarrier and raise the bytes its current phase waits for.
__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// try_wait with cluster-scope acquire: what other CTAs of the cluster wrote before their
// arrivals (or stored with complete_tx on this barrier) is visible once it returns true.
__device__ inline bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u) : "memory");
    return ok != 0;
}

// mbar_wait for a barrier that other CTAs of the cluster arrive on.
__device__ inline bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, unsigned epoch) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (timed_out_since(epoch)) return false;
        if (clock64() - t0 > kWaitLimitCycles) { raise_timeout(); return false; }
    }
    return true;
}

// Every thread of every CTA of the cluster (all of them must execute it).
__device__ inline void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// ------------------------------------------------------------------ PTX: cp.async

__device__ inline void cp_async_16(uint32_t dst_smem, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_smem), "l"(src) : "memory");
}
// Waits until every cp.async this thread has issued has landed, committed to a group or not
// (the gathers signal through mbarriers and are never committed; wait_group would skip them).
__device__ inline void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Arrive on `bar` (without raising its expected count) once every cp.async this thread has
// issued so far has landed in shared memory.
__device__ inline void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy
// (tcgen05.mma operand reads).
__device__ inline void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ PTX: tcgen05

__device__ inline void tmem_alloc(uint32_t* dst_smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem_slot)), "r"(ncols) : "memory");
}
__device__ inline void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ inline void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ inline void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ inline void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on `bar` once all tcgen05 operations issued so far by this thread complete.
__device__ inline void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 in, fp32 accumulate).
__device__ inline void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                   uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16: A (M x K, bf16 pairs packed per 32-bit
// column, row m in lane m) is read from tensor memory.
__device__ inline void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                   uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ inline void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ inline void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane (base + t).
__device__ inline void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ inline void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
          "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
          "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns, thread t of the warp writes lane (base + t).
__device__ inline void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// ---------------------------------------------------------- UMMA descriptors

// Shared-memory matrix descriptor for a 128-byte-swizzled tile (sm_100 format: start
// address, leading and stride byte offsets in 16-byte units, version 1, layout type 2).
__device__ inline uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t desc = 0;
    desc |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    desc |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    desc |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    desc |= (uint64_t)1 << 46;                 // descriptor version for sm_100
    desc |= (uint64_t)2 << 61;                 // SWIZZLE_128B
    return desc;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D, dense.
//   a_mn / b_mn: operand is MN-major (1) or K-major (0).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                    // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((uint32_t)a_mn << 15)
         | ((uint32_t)b_mn << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of 16-byte chunk `c` of row `r` in a K-major 128B-swizzled tile of `rows`
// rows: 64 bf16 columns per swizzle panel, panels stacked every rows*128 bytes.
__host__ __device__ inline uint32_t sw128_offset(int rows, int r, int c) {
    return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

}  // namespace bsa
