// kda_sm100.cuh -- sm_100a building blocks used by the KDA kernels: mbarriers,
// bulk (TMA-engine) copies, tcgen05 tensor-core MMA with TMEM accumulators,
// shared-memory matrix descriptors, bf16 helpers and bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define KDA_DEV __device__ __forceinline__

namespace kda {

// ----------------------------------------------------------------- status --
// Device status word (first 4 bytes of a chunk-forward workspace).  Bits are
// OR-ed in by kernels that detect a problem; the host reads them back with
// kda_query_status.
enum : uint32_t {
    DEV_ERR_TIMEOUT = 1u,   // a bounded mbarrier wait expired
    DEV_ERR_SEQLEN = 2u,    // cu_seqlens inconsistent with T or max_seqlen
};

// Wall-clock bound of one wait (%globaltimer is in ns): about one second.
constexpr unsigned long long WAIT_LIMIT_NS = 1000000000ull;

KDA_DEV uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

KDA_DEV unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier --
KDA_DEV void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

KDA_DEV void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

KDA_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Plain arrival (count 1) on a local mbarrier, release semantics at CTA scope.
KDA_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Tests the phase with the given parity; while it is incomplete the thread
// may be suspended in hardware for up to `suspend_ns` (so waiting warps do not
// consume issue slots) before the test returns false.
KDA_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t suspend_ns = 1000000u) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete.  Gives up after about
// limit_ns (WAIT_LIMIT_NS by default), ORs DEV_ERR_TIMEOUT into *status (if
// non-null) and returns false; never spins forever.
KDA_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                       unsigned long long limit_ns = WAIT_LIMIT_NS) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity, 100000u)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            if (status) atomicOr(status, DEV_ERR_TIMEOUT);
            return false;
        }
    }
}

// Same bound, but polling with mbarrier.test_wait instead of letting the hardware
// suspend the thread: a suspended waiter resumes later than a polling one sees the
// phase complete (about 50 cycles per wait in the chunk-local forward kernel, measured
// as its run time), which matters on a critical path of short waits (a CTA's own
// tensor-core products); use it where the waiting warps have nothing else to issue.
KDA_DEV bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
KDA_DEV bool mbar_wait_spin(uint64_t* bar, uint32_t parity, uint32_t* status,
                            unsigned long long limit_ns = WAIT_LIMIT_NS) {
    if (mbar_test_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((n & 255u) == 0 && globaltimer_ns() - t0 > limit_ns) {
            if (status) atomicOr(status, DEV_ERR_TIMEOUT);
            return false;
        }
    }
}

// ------------------------------------------- programmatic dependent launch --
// A kernel launched with programmatic stream serialisation may be scheduled before
// the kernel ahead of it in the stream has finished; pdl_wait() returns once that
// kernel has completed and its memory operations are visible, and must come before
// anything that reads what it writes.  pdl_trigger() in the earlier kernel lets the
// later one be scheduled as soon as every CTA has issued it (or exited).  Both are
// no-ops when the launches are not paired this way.
KDA_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
KDA_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------- bulk copies (TMA engine) --
// 1-D bulk copy global -> shared, completion signalled on `bar` (tx bytes).
// Both addresses 16-byte aligned, bytes a multiple of 16.
KDA_DEV void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Brings a tensor map (kernel parameter or global) into the descriptor cache.
KDA_DEV void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled TMA load of box (x, y) of a tensor map into shared memory,
// completion signalled on `bar`.  x is the innermost coordinate (elements);
// x * element size must be a multiple of 16 bytes.
KDA_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy shared -> global (bulk async-group completion).
KDA_DEV void bulk_s2g(void* gmem_dst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
                 "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}
KDA_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
KDA_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
KDA_DEV void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Makes generic-proxy shared-memory writes visible to the async proxy (tensor
// core operand reads, bulk copies).  Call before the barrier that precedes
// the MMA issue.
KDA_DEV void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// --------------------------------------------------------------- clusters --
KDA_DEV uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
KDA_DEV uint32_t map_to_cta(uint32_t local_smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem_addr), "r"(rank));
    return r;
}
// Asynchronous 4-byte store into (possibly another CTA's) shared memory; its
// arrival performs complete_tx(4) on the mbarrier at `cluster_bar_addr` in the
// destination CTA, so the receiver learns of it without any fence here.
KDA_DEV void st_async_f32(uint32_t cluster_addr, float v, uint32_t cluster_bar_addr) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];" ::"r"(cluster_addr),
                 "f"(v), "r"(cluster_bar_addr)
                 : "memory");
}
// Waits with acquire at cluster scope, polling (test_wait: the peers' partial sums are
// on the chain's critical path), bounded like mbar_wait.
KDA_DEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t* status) {
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
        if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
            if (status) atomicOr(status, DEV_ERR_TIMEOUT);
            return false;
        }
    }
}
KDA_DEV void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// sigmoid(x) = 0.5 tanh(x / 2) + 0.5 with the hardware tanh approximation (one
// special-function operation; relative error of tanh.approx about 2^-11).
KDA_DEV float sigmoid_fast(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}

// ---------------------------------------------------------------- tcgen05 --
// TMEM allocation: one warp allocates `ncols` columns (power of 2, >= 32) and
// the base address is written to *dst (shared memory).
KDA_DEV void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
KDA_DEV void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
KDA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
KDA_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
KDA_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 operands, fp32 accumulate).
// Issued by a single thread.
KDA_DEV void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on `bar` when all previously issued tcgen05.mma of this thread
// have completed.
KDA_DEV void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Instruction descriptor for kind::f16: bf16 A and B, fp32 D, both operands
// K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4)                         // D format: f32
           | (1u << 7)                       // A format: bf16
           | (1u << 10)                      // B format: bf16
           | ((uint32_t)(N >> 3) << 17)      // N / 8
           | ((uint32_t)(M >> 4) << 24);     // M / 16
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// 128-byte-swizzle canonical layout: rows of 128 bytes (64 bf16 along K),
// groups of 8 rows 1024 bytes apart, 16-byte chunk index XOR-ed with the row
// index within its 8-row group.  The operand region must be 1024-byte
// aligned; `addr` may be advanced by multiples of 32 bytes inside a 128-byte
// row to step K by 16 elements.
KDA_DEV uint64_t sdesc_k_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)(16u >> 4) << 16;                  // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset: 8-row group pitch
    d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                          // layout: SWIZZLE_128B
    return d;
}

// Shared-memory matrix descriptor for an operand in the no-swizzle
// ("interleaved") canonical layout: core matrices of 8 rows x 16 bytes, each
// 128 contiguous bytes.  For a K-major operand a core-matrix row runs along K;
// for an MN-major operand it runs along M/N.  lbo = byte distance between core
// matrices adjacent along K, sbo = between core matrices adjacent along M/N.
KDA_DEV uint64_t sdesc_interleave(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
    return d;                                         // layout: SWIZZLE_NONE (0)
}

// Instruction descriptor for kind::f16 (bf16 in, fp32 accumulate) with the
// operand majorness given: a_mn / b_mn = 1 for an MN-major operand.
__host__ __device__ constexpr uint32_t idesc_bf16_major(int M, int N, int a_mn, int b_mn) {
    return idesc_bf16(M, N) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16);
}

// Byte offset of element (mn, k) of an MN-major no-swizzle image whose core
// matrices are laid out with M/N-block stride 128 B and K-group stride
// kgroup_bytes (= 16 * MN extent): 8 consecutive mn form one 16-byte row.
__host__ __device__ __forceinline__ uint32_t mn_off(uint32_t mn, uint32_t k, uint32_t kgroup_bytes) {
    return (mn >> 3) * 128u + (k >> 3) * kgroup_bytes + (k & 7u) * 16u + (mn & 7u) * 2u;
}

// Byte offset of element (row, k) inside one 128-byte-wide K block of a
// K-major SW128 operand image (2-byte elements, k in [0, 64)).
__host__ __device__ __forceinline__ uint32_t sw128_off(uint32_t row, uint32_t k) {
    return row * 128u + ((((k >> 3) ^ (row & 7u)) & 7u) << 4) + ((k & 7u) << 1);
}

// TMEM load: 32 lanes x 32 bits, N consecutive columns per thread.
KDA_DEV void tmem_ld32(uint32_t taddr, float* r) {
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
          "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]),
          "=r"(u[22]), "=r"(u[23]), "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]),
          "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
}
KDA_DEV void tmem_ld16(uint32_t taddr, float* r) {
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
          "=r"(u[15])
        : "r"(taddr));
}
KDA_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// TMEM address of (lane, column) relative to an allocation base.
KDA_DEV uint32_t taddr(uint32_t base, uint32_t lane, uint32_t col) { return base + (lane << 16) + col; }

// ------------------------------------------------------------------- bf16 --
KDA_DEV float bf16_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }
KDA_DEV uint16_t f32_to_bf16(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
// Two floats -> one 32-bit word of two bf16 (round to nearest even), one
// paired conversion; `lo` lands in the low half.
KDA_DEV uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Loads one element of an input tensor stored as fp32 or bf16.
template <bool BF16>
KDA_DEV float ld_in(const void* base, size_t idx) {
    if constexpr (BF16) {
        return bf16_to_f32(__ldg(reinterpret_cast<const unsigned short*>(base) + idx));
    } else {
        return __ldg(reinterpret_cast<const float*>(base) + idx);
    }
}

template <bool BF16>
KDA_DEV void st_out(void* base, size_t idx, float v) {
    if constexpr (BF16) {
        reinterpret_cast<unsigned short*>(base)[idx] = f32_to_bf16(v);
    } else {
        reinterpret_cast<float*>(base)[idx] = v;
    }
}

constexpr float LOG_ALPHA_FLOOR = -5.0f;

}  // namespace kda
