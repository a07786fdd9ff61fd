// Thin helpers around the sm_100a 5th-generation tensor-core instructions
// (tcgen05.*): shared-memory matrix descriptors for 128-byte-swizzled bf16
// operands, the instruction descriptor for bf16 x bf16 -> fp32, TMEM
// allocation, MMA issue/commit, TMEM loads, bulk (TMA) global -> shared
// copies, and mbarrier waits that give up after a bounded time.
//
// Operand layouts (bf16, 128-byte swizzle; every tile base 1024-byte aligned):
//  * K-major tile of R rows (R % 8 == 0) and K columns: atom column kb = k / 64
//    holds R rows of 128 bytes; rows are grouped by 8 (1024 bytes). Within a
//    row the 16-byte chunk index is XOR-ed with (row % 8).
//      offset(r, k) = kb*R*128 + (r/8)*1024 + (r%8)*128 + (((k%64)/8) ^ (r%8))*16 + (k%8)*2
//    Descriptor: LBO = 16 B, SBO = 1024 B; the 16-element k-step ks starts at
//    base + (ks/4)*R*128 + (ks%4)*32.
//  * MN-major tile (N contiguous) of K rows and N columns (N % 64 == 0): atoms
//    of 8 k-rows x 64 n-elements (1024 bytes), laid out [k/8][n/64][k%8][128 B].
//      offset(k, n) = (k/8)*(N/64)*1024 + (n/64)*1024 + (k%8)*128 + (((n%64)/8) ^ (k%8))*16 + (n%8)*2
//    Descriptor: LBO = 1024 B (next 64 n), SBO = (N/64)*1024 B (next 8 k); the
//    k-step ks starts at base + 2*ks*SBO.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace lola {
namespace umma {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t kmajor_offset(int r, int k, int R)
{
    const int kb = k >> 6, kk = k & 63;
    return (uint32_t)(kb * R * 128 + (r >> 3) * 1024 + (r & 7) * 128 +
                      ((((kk >> 3) ^ (r & 7))) << 4) + ((kk & 7) << 1));
}

__device__ __forceinline__ uint32_t mnmajor_offset(int k, int n, int N)
{
    const int nb = n >> 6, nn = n & 63;
    return (uint32_t)((k >> 3) * (N >> 6) * 1024 + nb * 1024 + (k & 7) * 128 +
                      ((((nn >> 3) ^ (k & 7))) << 4) + ((nn & 7) << 1));
}

// Start of the 128-byte row that holds row r of 64-column block kb of a K-major
// tile (the row's 16-byte chunks are swizzled within it by the address).
__device__ __forceinline__ uint32_t kmajor_row(int r, int kb, int R)
{
    return (uint32_t)(kb * R * 128 + (r >> 3) * 1024 + (r & 7) * 128);
}
// Start of the 128-byte row that holds k-row k of 64-column block nb of an
// MN-major tile with N columns.
__device__ __forceinline__ uint32_t mnmajor_row(int k, int nb, int N)
{
    return (uint32_t)((k >> 3) * (N >> 6) * 1024 + nb * 1024 + (k & 7) * 128);
}

__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for sm_100
    d |= (uint64_t)2 << 61;   // 128-byte swizzle
    return d;
}

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int ks, int R)
{
    return make_desc(base + (uint32_t)((ks >> 2) * R * 128 + (ks & 3) * 32), 16, 1024);
}

__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int ks, int N)
{
    const uint32_t sbo = (uint32_t)(N >> 6) * 1024;
    return make_desc(base + (uint32_t)(2 * ks) * sbo, 1024, sbo);
}

// bf16 x bf16 -> fp32, dense; a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4)                     // D format fp32
           | (1u << 7)                   // A format bf16
           | (1u << 10)                  // B format bf16
           | ((a_mn ? 1u : 0u) << 15)    // A major
           | ((b_mn ? 1u : 0u) << 16)    // B major
           | ((uint32_t)(N >> 3) << 17)  // N / 8
           | ((uint32_t)(M >> 4) << 24); // M / 16
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; issued by one thread.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on an mbarrier once all previously issued MMAs of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t *mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :
                 : "r"(smem_u32(mbar))
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Makes generic-proxy shared-memory writes visible to the tensor core.
__device__ __forceinline__ void fence_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMEM allocation by one full warp; the base address lands in *slot (smem).
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :
                 : "r"(smem_u32(slot)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// 32 lanes x 16 consecutive fp32 columns: thread t of the warp gets lane
// (lane_base + t), columns [col, col + 16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 32 consecutive fp32 columns
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 columns store (thread t writes lane lane_base + t).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        :
        : "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
          "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
          "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
          "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
          "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
          "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t *mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)), "r"(count)
                 : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// One potentially blocking probe of an mbarrier phase (acquire, CTA scope): the
// thread sleeps until the phase completes or a hardware time slice runs out.
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    return done != 0;
}

// Probes between two looks at the clock (and the error word) while a wait is
// unfinished: a hand-off that completes within them costs no timer read and no
// global load.
constexpr int kProbesPerCheck = 16;

// Waits for the mbarrier phase `parity`; gives up after limit_ns nanoseconds of
// wall time (measured with %globaltimer) and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *mbar, uint32_t parity, uint64_t limit_ns)
{
    const uint32_t a = smem_u32(mbar);
    if (mbar_try(a, parity)) return true;
    const uint64_t start = globaltimer_ns();
    for (;;) {
        for (int k = 0; k < kProbesPerCheck; ++k)
            if (mbar_try(a, parity)) return true;
        if (globaltimer_ns() - start > limit_ns) return false;
    }
}

// One non-blocking probe of an mbarrier phase (acquire, CTA scope).
__device__ __forceinline__ bool mbar_test(uint64_t *mbar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(smem_u32(mbar)), "r"(parity)
        : "memory");
    return done != 0;
}

// As mbar_wait, but also gives up when *err holds a bit of abort_mask (another
// thread of the grid gave up). The error word, a global read, is only consulted
// between rounds of probes of an unfinished wait.
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t *mbar, uint32_t parity, uint64_t limit_ns,
                                                    const int *err, int abort_mask)
{
    const uint32_t a = smem_u32(mbar);
    if (mbar_try(a, parity)) return true;
    const uint64_t start = globaltimer_ns();
    for (;;) {
        for (int k = 0; k < kProbesPerCheck; ++k)
            if (mbar_try(a, parity)) return true;
        if ((*(const volatile int *)err & abort_mask) != 0) return false;
        if (globaltimer_ns() - start > limit_ns) return false;
    }
}

// Expects `bytes` more transaction bytes on the mbarrier and arrives once.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *mbar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(mbar)), "r"(bytes)
                 : "memory");
}

// Bulk (TMA, non-tensor) global -> shared copy of `bytes` (a multiple of 16;
// both addresses 16-byte aligned); completion is counted on the mbarrier.
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *mbar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :
        : "r"(smem_u32(smem_dst)), "l"(gmem_src), "r"(bytes), "r"(smem_u32(mbar))
        : "memory");
}

// Bulk (TMA, non-tensor) shared -> global copy, tracked as a bulk group of the
// issuing thread (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_s2g(void *gmem_dst, const void *smem_src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :
                 : "l"(gmem_dst), "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The shared-memory sources of this thread's bulk stores have been read.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// This thread's bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Tiled 3-D TMA load of one box into shared memory (no multicast); completion
// is counted on the mbarrier. tmap is the address of a __grid_constant__ map.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *tmap, int x, int y, int z, uint64_t *mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        :
        : "r"(smem_u32(smem_dst)), "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(mbar))
        : "memory");
}

// Tiled 2-D TMA load of one box (no multicast); completion counted on the mbarrier.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, int x, int y, uint64_t *mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :
        : "r"(smem_u32(smem_dst)), "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(mbar))
        : "memory");
}
// Orders this thread's generic-proxy global writes before later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Row gather (TMA tile::gather4, no multicast): rows r0..r3 of a 2-D row map,
// 64 columns from column x (x % 64 == 0), into four consecutive 128-byte rows
// at smem_dst (128-byte aligned; the 128-byte swizzle follows the address).
// Rows past the map's extent read as zero. Completion is counted on the mbarrier.
__device__ __forceinline__ void gather4(void *smem_dst, const void *tmap, int x, int r0, int r1, int r2, int r3,
                                        uint64_t *mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];"
        :
        : "r"(smem_u32(smem_dst)), "l"(tmap), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(mbar))
        : "memory");
}

// ---- thread-block clusters (distributed shared memory)
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t cluster_map(const void *local, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// arrive (release, cluster scope) on an mbarrier of another CTA of the cluster
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t remote_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
// one potentially blocking probe with cluster-scope acquire (pairs with mbar_arrive_cluster)
__device__ __forceinline__ bool mbar_try_cluster(uint32_t a, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    return done != 0;
}
// bounded wait with cluster-scope acquire
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *mbar, uint32_t parity, uint64_t limit_ns)
{
    const uint32_t a = smem_u32(mbar);
    if (mbar_try_cluster(a, parity)) return true;
    const uint64_t start = globaltimer_ns();
    for (;;) {
        for (int k = 0; k < kProbesPerCheck; ++k)
            if (mbar_try_cluster(a, parity)) return true;
        if (globaltimer_ns() - start > limit_ns) return false;
    }
}
// mbar_wait_cluster that also gives up when *err holds a bit of abort_mask; the error
// word is only read between rounds of probes of an unfinished wait
__device__ __forceinline__ bool mbar_wait_cluster_abortable(uint64_t *mbar, uint32_t parity, uint64_t limit_ns,
                                                            const int *err, int abort_mask)
{
    const uint32_t a = smem_u32(mbar);
    if (mbar_try_cluster(a, parity)) return true;
    const uint64_t start = globaltimer_ns();
    for (;;) {
        for (int k = 0; k < kProbesPerCheck; ++k)
            if (mbar_try_cluster(a, parity)) return true;
        if ((*(const volatile int *)err & abort_mask) != 0) return false;
        if (globaltimer_ns() - start > limit_ns) return false;
    }
}
// full cluster barrier (every thread of every CTA of the cluster)
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void fence_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// 2^x by the hardware approximation (ex2.approx, flush-to-zero)
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two fp32 -> one register holding two bf16 (round to nearest even); lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16lo_to_f32(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// 16-byte asynchronous global -> shared copy (L2 only).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
}
// 16-byte asynchronous copy of `bytes` (0 or 16) source bytes; the rest of the 16
// destination bytes are zero (src must still be a valid address)
__device__ __forceinline__ void cp_async16_zfill(void *smem, const void *gmem, uint32_t bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(bytes)
                 : "memory");
}
// Arrive (without raising the expected count) on the mbarrier once every cp.async this
// thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *mbar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(mbar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait_n() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// Programmatic dependent launch: the grid launched after this one on the stream (with
// programmatic stream serialisation) may start once every CTA of this grid executed this.
__device__ __forceinline__ void griddep_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Waits until the grid this one depends on (programmatic stream serialisation) has
// completed and its memory operations are visible; returns at once otherwise.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Plain arrive (count 1) on an mbarrier.
__device__ __forceinline__ void mbar_arrive(uint64_t *mbar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(mbar)) : "memory");
}

}  // namespace umma
}  // namespace lola
