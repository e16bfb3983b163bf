// sm100_ptx.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// EQ-Linear forward uses: mbarriers, TMA / bulk copies, tcgen05 (UMMA + TMEM).
//
// Descriptor bit layouts follow the PTX ISA "tcgen05 shared memory descriptor" and
// "instruction descriptor" tables.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace eqlin {
namespace ptx {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Dynamic shared memory rounded up to a 1 KB boundary by pointer arithmetic on the
// __shared__ array itself.  Every pointer derived from the result stays in the shared
// state space, so the compiler emits shared-memory loads and stores for it; rounding
// through an integer would turn all of them into generic accesses.
__device__ __forceinline__ uint8_t* smem_align_1k(uint8_t* raw) {
    return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
        "r"(bytes)
        : "memory");
}
// true once the phase with the given parity has completed
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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
// Same test, but a thread whose phase is not complete is suspended (it stops taking
// issue slots from the warps doing work) until the phase completes or `hint_ns`
// elapses, whichever comes first.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------ programmatic dependent launch
// Let the next kernel of the stream (launched with programmatic stream serialization)
// start launching its CTAs now.
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Block until the preceding kernel of the stream has completed and its memory
// operations are visible (a no-op when this kernel was not launched as a dependent).
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ------------------------------------------------------------ CTA barriers
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Barrier over `nthreads` threads that also ANDs a predicate across them.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------------ async copies
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 2-D tiled TMA load global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, int32_t c0,
                                            int32_t c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
// 2-D tiled TMA store shared -> global (bulk async-group completion).  Rows or columns
// of the box outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, uint32_t src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(src)
                 : "memory");
}
// L2 eviction-priority policies for the cache-hinted copies below: data read again soon
// (weights shared by every CTA) is kept in L2 before data streamed once (x, y).
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// tma_load_2d with an L2 cache policy
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* m, int32_t c0, int32_t c1,
                                                 uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
        : "memory");
}
// tma_store_2d with an L2 cache policy
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* m, uint32_t src, int32_t c0, int32_t c1,
                                                  uint64_t policy) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%1, %2}], [%3], %4;" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(src), "l"(policy)
                 : "memory");
}
// Hint: bring the 2-D box at (c0, c1) of the tensor into L2 (no shared memory, no
// completion to wait for; parts of the box outside the tensor are not fetched).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* m, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N committed bulk groups of this thread are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Plain bulk copy global -> shared (16-B aligned addresses, size multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// bulk_load with an L2 cache policy
__device__ __forceinline__ void bulk_load_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                               uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}
// The copies above with an optional L2 policy (hint == false: the plain form).
__device__ __forceinline__ void bulk_load_h(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar, bool hint,
                                            uint64_t policy) {
    if (hint) bulk_load_hint(dst, src, bytes, bar, policy);
    else bulk_load(dst, src, bytes, bar);
}
__device__ __forceinline__ void tma_load_2d_h(uint32_t dst, const CUtensorMap* m, int32_t c0, int32_t c1, uint32_t bar,
                                              bool hint, uint64_t policy) {
    if (hint) tma_load_2d_hint(dst, m, c0, c1, bar, policy);
    else tma_load_2d(dst, m, c0, c1, bar);
}
__device__ __forceinline__ void tma_store_2d_h(const CUtensorMap* m, uint32_t src, int32_t c0, int32_t c1, bool hint,
                                               uint64_t policy) {
    if (hint) tma_store_2d_hint(m, src, c0, c1, policy);
    else tma_store_2d(m, src, c0, c1);
}
// Make this thread's generic-proxy shared-memory writes visible to the async proxy
// (tensor-core operand reads, later TMA writes).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ tcgen05 / TMEM
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
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive (once) on `bar` when every tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Ties registers filled by tcgen05.ld to a preceding tmem_wait_ld(): an empty volatile
// asm per register stays ordered after the wait, and every later use of the register
// depends on it, so no use can be scheduled before the data is valid.
template <int N>
__device__ __forceinline__ void tmem_regs_ready(uint32_t (&r)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// 32 lanes x 32 bits x N consecutive columns: thread t gets lane (base+t), columns [col, col+N).
template <int N>
__device__ __forceinline__ void tmem_ld_32x32b(uint32_t taddr, uint32_t (&r)[N]);

template <>
__device__ __forceinline__ void tmem_ld_32x32b<2>(uint32_t taddr, uint32_t (&r)[2]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_32x32b<4>(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_32x32b<8>(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_32x32b<16>(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_32x32b<32>(uint32_t taddr, uint32_t (&r)[32]) {
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
}

// --------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor, K-major operand with 64-byte swizzle:
// rows of 64 B (32 bf16 along K), 8-row atoms of 512 B, atoms stacked along
// M/N at 512 B.  start: shared address of the first row (16-B granular).
__device__ __forceinline__ uint64_t sdesc_kmajor_sw64(uint32_t start) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((start & 0x3FFFFu) >> 4);  // bits [0,14): start >> 4
    d |= static_cast<uint64_t>(1) << 16;                 // [16,30): LBO, unused for swizzled K-major
    d |= static_cast<uint64_t>(512 >> 4) << 32;          // [32,46): SBO = 512 B between 8-row groups
    d |= static_cast<uint64_t>(1) << 46;                 // [46,48): descriptor version 1 (sm_100)
    d |= static_cast<uint64_t>(4) << 61;                 // [61,64): layout 4 = SWIZZLE_64B
    return d;                                            // base offset 0, LBO mode 0
}

// K-major operand with 32-byte swizzle: rows of 32 B (16 bf16 along K = one MMA K
// step), 8-row atoms of 256 B stacked along M/N.
__device__ __forceinline__ uint32_t sdesc_sw32_lo(uint32_t start) { return (1u << 16) | (start >> 4); }
constexpr uint32_t kSdescSw32Hi = (256u >> 4) | (1u << 14) | (6u << 29);
__device__ __forceinline__ uint64_t sdesc_sw32_from_lo(uint32_t lo) {
    return (static_cast<uint64_t>(kSdescSw32Hi) << 32) | lo;
}

// The same descriptor split in halves: only the start-address field (low 14 bits)
// varies between operands, so the issuing loop adds (byte offset >> 4) to the low
// half and pairs it with the constant high half.
__device__ __forceinline__ uint32_t sdesc_sw64_lo(uint32_t start) { return (1u << 16) | (start >> 4); }
constexpr uint32_t kSdescSw64Hi = (512u >> 4) | (1u << 14) | (4u << 29);
__device__ __forceinline__ uint64_t sdesc_sw64_from_lo(uint32_t lo) {
    return (static_cast<uint64_t>(kSdescSw64Hi) << 32) | lo;
}

// MN-major operand with 64-byte swizzle: each 8-row atom (512 B) holds 8 consecutive
// K indices as rows of 64 B = 32 consecutive M (or N) elements; lbo = byte stride
// between atoms along M/N, sbo = byte stride between 8-row groups along K.  Split in
// halves like the K-major forms: the high half carries sbo, version and layout.
__device__ __forceinline__ uint32_t sdesc_mn_sw64_lo(uint32_t start, uint32_t lbo) {
    return ((lbo >> 4) << 16) | (start >> 4);
}
__device__ __forceinline__ uint32_t sdesc_mn_sw64_hi(uint32_t sbo) {
    return ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (4u << 29);
}
__device__ __forceinline__ uint64_t sdesc_from_halves(uint32_t hi, uint32_t lo) {
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

}  // namespace ptx

// Instruction descriptor for tcgen05.mma kind::f16 with an fp32 D, both operands
// K-major.  fmt is the A and B operand format (0 F16, 1 BF16; A and B share it).
// M in {64,128}, N a multiple of 16 up to 256.
__host__ __device__ constexpr uint32_t idesc_f16kind_f32(int M, int N, uint32_t fmt, bool negate_a,
                                                         bool negate_b = false) {
    return (1u << 4)                                  // D format: F32
           | (fmt << 7)                               // A format
           | (fmt << 10)                              // B format
           | ((negate_a ? 1u : 0u) << 13)             // negate A
           | ((negate_b ? 1u : 0u) << 14)             // negate B
           | (static_cast<uint32_t>(N >> 3) << 17)    // N >> 3
           | (static_cast<uint32_t>(M >> 4) << 24);   // M >> 4
}

// the same with both operands MN-major (A: M contiguous, B: N contiguous)
__host__ __device__ constexpr uint32_t idesc_f16kind_f32_mn(int M, int N, uint32_t fmt, bool negate_a,
                                                            bool negate_b = false) {
    return idesc_f16kind_f32(M, N, fmt, negate_a, negate_b) | (1u << 15) | (1u << 16);
}

// bf16 A and B
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool negate_a, bool negate_b = false) {
    return idesc_f16kind_f32(M, N, 1u, negate_a, negate_b);
}

}  // namespace eqlin
