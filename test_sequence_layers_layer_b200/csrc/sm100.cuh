// sm100.cuh -- thin inline-PTX layer for the Blackwell (sm_100a) features
// used by the tensor-core kernels: shared-memory mbarriers with bounded waits,
// tensor memory (TMEM) allocation / load, tcgen05.mma with shared-memory
// matrix descriptors, and the canonical operand layouts those descriptors
// describe. Written from the PTX ISA's description of tcgen05.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ttt {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// Makes initialised mbarriers visible to the async proxy (tensor core, TMA).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Suspend-time hint of one try_wait (ns): a waiting warp is parked by the
// hardware until the phase completes or the hint elapses, instead of spinning
// and taking issue slots from the warps doing the work.
constexpr uint32_t kTryWaitSuspendNs = 1000000;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kTryWaitSuspendNs)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Upper bound of any single wait on an on-chip barrier. A correct kernel
// waits microseconds; running out means a protocol bug, and the kernel then
// records it and unwinds instead of hanging the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Retry loop of mbar_wait, kept out of line: the first try_wait (which parks
// the warp until the phase completes) nearly always succeeds, and inlining
// the loop at every wait site would multiply the kernels' code size.
static __device__ __noinline__ bool mbar_wait_slow(uint32_t a, uint32_t parity,
                                                   volatile int *abort, int *status, int code,
                                                   uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(a, parity)) return true;
        if ((i & 3u) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort = 1;
                if (status) atomicExch(status, code);
                return false;
            }
        }
    }
}

// Waits for phase `parity` of the mbarrier to complete. On timeout sets
// *abort (shared flag seen by the whole block), records `code` in the
// device status word and returns false. Returns false at once if another
// thread already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          int *status, int code,
                                          uint64_t limit_ns = kWaitLimitNs) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    return mbar_wait_slow(a, parity, abort, status, code, limit_ns);
}

// Arrive and add `bytes` to the transaction count the phase waits for.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Like mbar_wait but ignores the abort flag: used while unwinding after an
// abort, to let this thread's own in-flight copies or MMAs land first.
__device__ __forceinline__ bool mbar_drain(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(a, parity)) return true;
        if ((i & 3u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// ----------------------------------------------------------------- TMA

// 2-D tiled bulk tensor load global -> shared, completing on `bar`
// (transaction bytes). x is the innermost coordinate (elements).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Contiguous bulk copy global -> shared (no tensor map), completing on `bar`.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Bulk prefetch of global memory into L2 (a hint: nothing waits for it).
// Address 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)),
                 "r"(bytes)
                 : "memory");
}

// Contiguous bulk copy shared -> global (async proxy), tracked by the issuing
// thread's bulk async-groups (bulk_commit, bulk_wait_read, bulk_wait). Both
// addresses 16-byte aligned, size a multiple of 16; the shared source is
// written before a fence.proxy.async.shared::cta (fence_async_smem).
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                     reinterpret_cast<uint64_t>(dst)),
                 "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// All but the newest N groups have finished reading their shared sources.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// All but the newest N groups are complete (their writes performed).
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ----------------------------------------------------------------- fences

// Generic-proxy writes to shared memory -> visible to the async proxy (MMA).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ----------------------------------------------------------------- TMEM

// Warp-collective: allocates `ncols` (power of two >= 32) TMEM columns and
// writes the base address to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// TMEM address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t taddr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// Warp-collective 32-lane x 32-bit load, 16 consecutive columns: thread i
// receives columns col..col+15 of lane (base lane + i). The warp may only
// address the 32 lanes of its own subpartition (warp id % 4).
__device__ __forceinline__ void tmem_ld16(uint32_t ta, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(ta));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Warp-collective load of the first 16 lanes of the subpartition, twice:
// thread i < 16 receives columns col..col+15 of lane (base lane + i), thread
// 16 + i the columns col+kSplit..col+kSplit+15 of the same lane. For an
// M = 64 accumulator (16 lanes per subpartition) this keeps all 32 threads busy.
template <int kSplit>
__device__ __forceinline__ void tmem_ld16_x2(uint32_t ta, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], %17;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(ta), "n"(kSplit));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Warp-collective 32-lane x 32-bit store of 16 consecutive columns (the
// mirror of tmem_ld16).
__device__ __forceinline__ void tmem_st16(uint32_t ta, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(ta),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Named barrier over `nthreads` threads (multiple of 32), id 1..15, that
// also returns the OR of every participant's `v` (so a group can agree to
// leave a loop together).
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// mbar_wait by every lane of a warp, with the warp agreeing on the outcome
// (keeps warp-collective instructions after it converged).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort,
                                               int *status, int code) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status, code));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ----------------------------------------------------------------- MMA

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"):
// start address, leading- and stride-dimension byte offsets (16-byte units),
// descriptor version 1, swizzle mode.
enum Swizzle : uint32_t { kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6 };

__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes, Swizzle sw) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;  // version 1 (Blackwell)
    d |= (uint64_t)sw << 61;
    return d;
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulator.
// a_mn / b_mn: operand stored MN-major (transposed) instead of K-major.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                      // D format f32
           | (1u << 7)                    // A format bf16
           | (1u << 10)                   // B format bf16
           | ((a_mn ? 1u : 0u) << 15)     // A major
           | ((b_mn ? 1u : 0u) << 16)     // B major
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: A (M x 16 per instruction for bf16) is read
// from tensor memory, row m in lane m, two K values per 32-bit column (the
// even one in the low half), 8 columns per instruction; B by descriptor.
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                                uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// Arrive once on the mbarrier when every MMA issued so far by this thread has
// completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// ----------------------------------------------------------------- layouts
// Byte offsets of element (row, col) of a bf16 operand tile in the canonical
// shared-memory layouts the descriptors above describe. "K-major" tiles are
// indexed (mn, k); "MN-major" tiles are indexed (k, mn), the contiguous index
// last. Tile bases must be 1024-byte aligned for the 128-byte swizzle.

// 128-byte swizzle, K-major: 8-row x 128-byte atoms (64 bf16 of K per row);
// atoms stacked along MN every 1024 bytes; for K > 64 the next 64 columns
// start after all MN rows (mn_rows * 128 bytes). SBO = 1024.
__host__ __device__ __forceinline__ uint32_t off_kmajor_sw128(uint32_t mn, uint32_t k,
                                                              uint32_t mn_rows) {
    const uint32_t kb = k >> 6, kk = k & 63;
    return kb * mn_rows * 128u + (mn >> 3) * 1024u + (mn & 7) * 128u +
           ((((kk * 2) >> 4) ^ (mn & 7)) << 4) + (kk & 7) * 2;
}

// 128-byte swizzle, MN-major: 8-row (K) x 128-byte (64 MN elements) atoms;
// 8-row groups along K every 1024 bytes (SBO); for MN > 64 the next 64 columns
// start after all K rows (k_rows * 128 bytes = LBO).
__host__ __device__ __forceinline__ uint32_t off_mnmajor_sw128(uint32_t k, uint32_t mn,
                                                               uint32_t k_rows) {
    const uint32_t mb = mn >> 6, mm = mn & 63;
    return mb * k_rows * 128u + (k >> 3) * 1024u + (k & 7) * 128u +
           ((((mm * 2) >> 4) ^ (k & 7)) << 4) + (mm & 7) * 2;
}

// No swizzle, K-major ("interleaved"): 8x8 core matrices of 16-byte rows;
// the two 8-column halves of a 16-wide K step are LBO = 128 bytes apart and
// 8-row groups are SBO = k_cols * 16 bytes apart.
__host__ __device__ __forceinline__ uint32_t off_kmajor_none(uint32_t mn, uint32_t k,
                                                             uint32_t k_cols) {
    return (mn >> 3) * (k_cols * 16u) + (k >> 3) * 128u + (mn & 7) * 16u + (k & 7) * 2;
}

// Split an fp32 value into two bf16 whose sum carries ~16 significant bits:
// hi = RN(x), lo = RN(x - hi).
// Two-term bf16 split of a pair: hi = x with the low 16 bits cleared (exact
// bf16, |x - hi| < 2^-7 |x|), lo = RN_bf16(x - hi); hi + lo carries ~16
// significant bits. Returns the packed hi pair and lo pair.
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const uint32_t ua = __float_as_uint(a) & 0xFFFF0000u, ub = __float_as_uint(b) & 0xFFFF0000u;
    hi = __byte_perm(ua, ub, 0x7632);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - __uint_as_float(ua), b - __uint_as_float(ub));
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

}  // namespace sm100
}  // namespace ttt

// ----------------------------------------------------------------- warp-level MMA
// m16n8k16 bf16 MMA with fp32 accumulation, issued by one warp, operands in
// registers. Fragment ownership (g = lane / 4, q = lane % 4; a register holds
// two bf16, the lower column in the low half):
//   A (16x16, row-major): a0 = A[g][2q..2q+1], a1 = A[g+8][2q..], a2 = A[g][2q+8..], a3 = A[g+8][2q+8..]
//   B (16x8):             b0 = B[2q..2q+1][g], b1 = B[2q+8..2q+9][g]
//   D (16x8):             d0 = D[g][2q], d1 = D[g][2q+1], d2 = D[g+8][2q], d3 = D[g+8][2q+1]
// Two side-by-side D tiles of a 16x16 matrix, packed pairwise, are that
// matrix's A fragment; movmatrix transposes an 8x8 block between the
// row-pair layouts of A/D and the column-pair layout of B.
namespace ttt {
namespace sm100 {

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 b16 block held one row-pair per lane.
__device__ __forceinline__ uint32_t movt(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// ldmatrix: lanes 8i..8i+7 give the shared addresses of the eight 16-byte
// rows of 8x8 b16 matrix i; each lane receives its row-pair of every matrix
// (.trans: of every matrix's transpose).
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

}  // namespace sm100
}  // namespace ttt

// ----------------------------------------------------------------- clusters
// Thread-block clusters: the CTA's rank, addresses of another CTA's shared
// memory (mapa), and the whole-cluster barrier.
namespace ttt {
namespace sm100 {

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address, in the cluster's shared window, of the variable at this CTA's
// shared address `a` in CTA `rank`.
__device__ __forceinline__ uint32_t mapa(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

// Whole-cluster barrier (every thread of every CTA), release/acquire.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

}  // namespace sm100
}  // namespace ttt

// ----------------------------------------------------------------- cluster bulk copies
namespace ttt {
namespace sm100 {

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// this CTA's shared memory to shared memory of a CTA of the cluster; the
// bytes count as completed transactions on the mbarrier `cluster_bar` (in
// the destination CTA). The writers of the source fence it for the async
// proxy first (fence_async_smem).
__device__ __forceinline__ void bulk_copy_to_cluster(uint32_t cluster_dst, uint32_t src,
                                                     uint32_t bytes, uint32_t cluster_bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            cluster_dst),
        "r"(src), "r"(bytes), "r"(cluster_bar)
        : "memory");
}

}  // namespace sm100
}  // namespace ttt

// ----------------------------------------------------------------- narrow TMEM loads
namespace ttt {
namespace sm100 {

// Warp-collective 32-lane x 32-bit load of 8 consecutive columns: thread i
// receives columns col..col+7 of lane (base lane + i).
__device__ __forceinline__ void tmem_ld8(uint32_t ta, float (&v)[8]) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(ta));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace sm100
}  // namespace ttt
