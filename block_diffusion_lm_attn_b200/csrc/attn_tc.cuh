// Building blocks of the tcgen05 block-diffusion attention kernel
// (attn_tc_persist.cuh): tile shapes and the shared-memory layout, mbarrier
// and TMA wrappers with bounded waits, tcgen05 MMA / TMEM load-store
// wrappers and descriptors, and the per-tile softmax pieces.
//
// Tiles: 128 query rows x 128 keys x head dim 128, bf16 operands, fp32
// accumulators in tensor memory (TMEM).  Q, K and V tiles are staged by TMA
// as two 64-column boxes with the 128-byte swizzle; S = Q K^T takes Q and K
// K-major from shared memory, O += P V takes P from TMEM and V MN-major from
// shared memory.
//
// Exactness of the lazy rescale used by the softmax: P_j = 2^(x - m_used)
// where m_used is the running maximum the row last rescaled to; it is raised
// (and O, l rescaled) only when the tile maximum exceeds m_used + 8, so
// P <= 2^8, and out = O / l and lse = (m_used + log2 l) ln 2 are exact for any
// m_used.
//
// Every mbarrier wait is bounded (kWaitCycles); a wait that runs out sets the
// CTA's abort flag and the device status word.
#pragma once

#include <cuda.h>

#include "bd_mask.cuh"
#include "bd_common.cuh"

namespace bd {

constexpr int kTcThreads = 224; // 4 softmax warps, K producer, MMA, V producer
constexpr int kTcM = 128;     // query rows per CTA
constexpr int kTcN = 128;     // keys per K/V tile
constexpr int kTcD = 128;     // head dim
constexpr int kTcStages = 2; // depth of the K ring and of the V ring
// TMEM S/P buffers of the persistent kernel (128 columns each; O takes the
// remaining 128 of the 512)
constexpr int kSBufs = 3;
#ifndef BD_EXP2_EMU
#define BD_EXP2_EMU 1
#endif
// evaluate a quarter of each tile's exponentials with ex2_poly2
constexpr bool kEmuExp2 = BD_EXP2_EMU != 0;
constexpr int kTileBytes = kTcN * kTcD * 2;          // 32 KB
constexpr int kHalfTileBytes = kTileBytes / 2;       // one 64-column box
#ifdef BD_TC_TRACE
// Debug builds only: per-CTA progress words in host-mapped memory, and short
// bounded waits, so a stalled launch shows which role stopped where.
constexpr long long kWaitCycles = 200000000LL;       // ~0.1 s at 2 GHz
__device__ uint32_t *g_tc_trace;
#define BD_TRACE(slot, val)                                                    \
    do {                                                                       \
        if (g_tc_trace) {                                                      \
            const int cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
            ((volatile uint32_t *)g_tc_trace)[cta_ * 8 + (slot)] = (val);      \
            __threadfence_system();                                            \
        }                                                                      \
    } while (0)
#else
constexpr long long kWaitCycles = 4000000000LL;      // ~2 s at 2 GHz
#define BD_TRACE(slot, val) do { } while (0)
#endif


// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int kSmemQ = 0;                      // two Q buffers
constexpr int kSmemK = kSmemQ + 2 * kTileBytes;
constexpr int kSmemV = kSmemK + kTcStages * kTileBytes;
// epilogue staging: per softmax warp, its 32 output rows of 256 bytes
constexpr int kSmemEpi = kSmemV + kTcStages * kTileBytes;
constexpr int kSmemBar = kSmemEpi + 4 * 32 * 256;
constexpr int kSmemSeg = kSmemBar + 512;                // 4 decoded work items, 128 B each
constexpr int kTcSmemBytes = kSmemSeg + 4 * 128 + 1024; // + alignment slack
static_assert(kTcSmemBytes <= 227 * 1024, "more shared memory than a CTA may have");

// ---------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar),
                 "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                     bar),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return ok != 0;
}

// As mbar_try_wait, but a thread whose phase has not completed is suspended
// in hardware until it completes or about `ns` nanoseconds pass, instead of
// spinning on the issue slots it shares with the other warps of its SM
// sub-partition.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t ns)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity), "r"(ns)
                 : "memory");
    return ok != 0;
}

#ifndef BD_WAIT_SLEEP_NS
#define BD_WAIT_SLEEP_NS 2000
#endif

// Bounded wait on phase `parity` of barrier `bar`.  Returns false if the
// CTA was aborted (by this wait running out or by another role).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, BD_WAIT_SLEEP_NS))
            return true;
        if (*abort_flag)
            return false;
        if (clock64() - t0 > kWaitCycles) {
            *abort_flag = 1;
            raise_device_code(DEV_WAIT_TIMEOUT);
            return false;
        }
    }
}

// mbar_wait by every lane of a converged warp; the result is the same in all
// lanes (false if any lane's wait gave up)
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile int *abort_flag)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *tm,
                                            int c0, int c1, int c2,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.mbarrier::complete_tx::"
        "bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2),
        "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::"
                 "cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc,
                                          uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(
                     d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem,
                                          uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(
                     d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// 1 in the one lane elect.sync picks in a converged warp, else 0
__device__ __forceinline__ uint32_t elect_one()
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "selp.u32 %0, 1, 0, e;\n\t}"
                 : "=r"(r));
    return r;
}
// tc_mma_ss / tc_mma_ts / tc_commit issued only where `leader` is nonzero,
// as a predicated instruction, so that a whole warp runs the issue loop
__device__ __forceinline__ void tc_mma_ss_p(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate, uint32_t leader)
{
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "setp.ne.b32 q, %5, 0;\n\t"
                 "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
                 : "memory");
}
__device__ __forceinline__ void tc_mma_ts_p(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate, uint32_t leader)
{
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "setp.ne.b32 q, %5, 0;\n\t"
                 "@q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
                 : "memory");
}
__device__ __forceinline__ void tc_commit_p(uint32_t bar, uint32_t leader)
{
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %1, 0;\n\t"
                 "@q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::"
                 "cluster.b64 [%0];\n\t}"
                 ::"r"(bar), "r"(leader)
                 : "memory");
}

// TMEM loads, shape 32x32b: thread i of the warp reads TMEM lane
// 32 * (warp id mod 4) + i, consecutive 32-bit columns from the address's
// column on; each is fused with its tcgen05.wait::ld in one statement.  The destination registers are defined
// only once the loads have landed, so the compiler can neither read them
// early nor spill them while a load is in flight; a separate load and wait
// would be correct only if nothing between the two touched the registers,
// which the compiler does not know.
// 32 columns
__device__ __forceinline__ void tmem_ld32_wait(uint32_t a0, uint32_t *r0)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
        "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31"
        "}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r0[0]), "=r"(r0[1]), "=r"(r0[2]), "=r"(r0[3]), "=r"(r0[4]),
          "=r"(r0[5]), "=r"(r0[6]), "=r"(r0[7]), "=r"(r0[8]), "=r"(r0[9]),
          "=r"(r0[10]), "=r"(r0[11]), "=r"(r0[12]), "=r"(r0[13]), "=r"(r0[14]),
          "=r"(r0[15]), "=r"(r0[16]), "=r"(r0[17]), "=r"(r0[18]), "=r"(r0[19]),
          "=r"(r0[20]), "=r"(r0[21]), "=r"(r0[22]), "=r"(r0[23]), "=r"(r0[24]),
          "=r"(r0[25]), "=r"(r0[26]), "=r"(r0[27]), "=r"(r0[28]), "=r"(r0[29]),
          "=r"(r0[30]), "=r"(r0[31])
        : "r"(a0)
        : "memory");
}
// two loads of 32 columns from a0 and a1
__device__ __forceinline__ void tmem_ld32x2_wait(uint32_t a0, uint32_t a1, uint32_t *r0, uint32_t *r1)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
        "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31"
        "}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63"
        "}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r0[0]), "=r"(r0[1]), "=r"(r0[2]), "=r"(r0[3]), "=r"(r0[4]),
          "=r"(r0[5]), "=r"(r0[6]), "=r"(r0[7]), "=r"(r0[8]), "=r"(r0[9]),
          "=r"(r0[10]), "=r"(r0[11]), "=r"(r0[12]), "=r"(r0[13]), "=r"(r0[14]),
          "=r"(r0[15]), "=r"(r0[16]), "=r"(r0[17]), "=r"(r0[18]), "=r"(r0[19]),
          "=r"(r0[20]), "=r"(r0[21]), "=r"(r0[22]), "=r"(r0[23]), "=r"(r0[24]),
          "=r"(r0[25]), "=r"(r0[26]), "=r"(r0[27]), "=r"(r0[28]), "=r"(r0[29]),
          "=r"(r0[30]), "=r"(r0[31]), "=r"(r1[0]), "=r"(r1[1]), "=r"(r1[2]),
          "=r"(r1[3]), "=r"(r1[4]), "=r"(r1[5]), "=r"(r1[6]), "=r"(r1[7]),
          "=r"(r1[8]), "=r"(r1[9]), "=r"(r1[10]), "=r"(r1[11]), "=r"(r1[12]),
          "=r"(r1[13]), "=r"(r1[14]), "=r"(r1[15]), "=r"(r1[16]), "=r"(r1[17]),
          "=r"(r1[18]), "=r"(r1[19]), "=r"(r1[20]), "=r"(r1[21]), "=r"(r1[22]),
          "=r"(r1[23]), "=r"(r1[24]), "=r"(r1[25]), "=r"(r1[26]), "=r"(r1[27]),
          "=r"(r1[28]), "=r"(r1[29]), "=r"(r1[30]), "=r"(r1[31])
        : "r"(a0), "r"(a1)
        : "memory");
}
// four loads of 32 columns from a0 .. a3
__device__ __forceinline__ void tmem_ld32x4_wait(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t *r0, uint32_t *r1, uint32_t *r2, uint32_t *r3)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
        "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31"
        "}, [%128];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63"
        "}, [%129];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
        "%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
        "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95"
        "}, [%130];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
        "%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
        "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127"
        "}, [%131];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r0[0]), "=r"(r0[1]), "=r"(r0[2]), "=r"(r0[3]), "=r"(r0[4]),
          "=r"(r0[5]), "=r"(r0[6]), "=r"(r0[7]), "=r"(r0[8]), "=r"(r0[9]),
          "=r"(r0[10]), "=r"(r0[11]), "=r"(r0[12]), "=r"(r0[13]), "=r"(r0[14]),
          "=r"(r0[15]), "=r"(r0[16]), "=r"(r0[17]), "=r"(r0[18]), "=r"(r0[19]),
          "=r"(r0[20]), "=r"(r0[21]), "=r"(r0[22]), "=r"(r0[23]), "=r"(r0[24]),
          "=r"(r0[25]), "=r"(r0[26]), "=r"(r0[27]), "=r"(r0[28]), "=r"(r0[29]),
          "=r"(r0[30]), "=r"(r0[31]), "=r"(r1[0]), "=r"(r1[1]), "=r"(r1[2]),
          "=r"(r1[3]), "=r"(r1[4]), "=r"(r1[5]), "=r"(r1[6]), "=r"(r1[7]),
          "=r"(r1[8]), "=r"(r1[9]), "=r"(r1[10]), "=r"(r1[11]), "=r"(r1[12]),
          "=r"(r1[13]), "=r"(r1[14]), "=r"(r1[15]), "=r"(r1[16]), "=r"(r1[17]),
          "=r"(r1[18]), "=r"(r1[19]), "=r"(r1[20]), "=r"(r1[21]), "=r"(r1[22]),
          "=r"(r1[23]), "=r"(r1[24]), "=r"(r1[25]), "=r"(r1[26]), "=r"(r1[27]),
          "=r"(r1[28]), "=r"(r1[29]), "=r"(r1[30]), "=r"(r1[31]), "=r"(r2[0]),
          "=r"(r2[1]), "=r"(r2[2]), "=r"(r2[3]), "=r"(r2[4]), "=r"(r2[5]),
          "=r"(r2[6]), "=r"(r2[7]), "=r"(r2[8]), "=r"(r2[9]), "=r"(r2[10]),
          "=r"(r2[11]), "=r"(r2[12]), "=r"(r2[13]), "=r"(r2[14]), "=r"(r2[15]),
          "=r"(r2[16]), "=r"(r2[17]), "=r"(r2[18]), "=r"(r2[19]), "=r"(r2[20]),
          "=r"(r2[21]), "=r"(r2[22]), "=r"(r2[23]), "=r"(r2[24]), "=r"(r2[25]),
          "=r"(r2[26]), "=r"(r2[27]), "=r"(r2[28]), "=r"(r2[29]), "=r"(r2[30]),
          "=r"(r2[31]), "=r"(r3[0]), "=r"(r3[1]), "=r"(r3[2]), "=r"(r3[3]),
          "=r"(r3[4]), "=r"(r3[5]), "=r"(r3[6]), "=r"(r3[7]), "=r"(r3[8]),
          "=r"(r3[9]), "=r"(r3[10]), "=r"(r3[11]), "=r"(r3[12]), "=r"(r3[13]),
          "=r"(r3[14]), "=r"(r3[15]), "=r"(r3[16]), "=r"(r3[17]), "=r"(r3[18]),
          "=r"(r3[19]), "=r"(r3[20]), "=r"(r3[21]), "=r"(r3[22]), "=r"(r3[23]),
          "=r"(r3[24]), "=r"(r3[25]), "=r"(r3[26]), "=r"(r3[27]), "=r"(r3[28]),
          "=r"(r3[29]), "=r"(r3[30]), "=r"(r3[31])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3)
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]),
        "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]),
        "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st()
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading
// and stride byte offsets (all >> 4), version 1, layout 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo,
                                                    uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46; // version
    d |= (uint64_t)2 << 61; // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, A
// K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn)
{
    return (1u << 4)      // D format: f32
           | (1u << 7)    // A format: bf16
           | (1u << 10)   // B format: bf16
           | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// (d0, d1) = (a0, a1) * (b0, b1) + (c0, c1), one packed instruction.
__device__ __forceinline__ void ffma2(float &d0, float &d1, float a0, float a1,
                                      float b0, float b1, float c0, float c1)
{
    asm("{\n\t.reg .b64 A, B, C, D;\n\t"
        "mov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
        "mov.b64 C, {%6, %7};\n\tfma.rn.f32x2 D, A, B, C;\n\t"
        "mov.b64 {%0, %1}, D;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
// (d0, d1) = (a0, a1) + (b0, b1), one packed instruction.
__device__ __forceinline__ void fadd2(float &d0, float &d1, float a0, float a1,
                                      float b0, float b1)
{
    asm("{\n\t.reg .b64 A, B, D;\n\t"
        "mov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
        "add.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// 2^x for a pair of x <= 8 on the FMA and integer pipes, leaving the
// special-function unit to the other exponentials of the tile.
// Cody-Waite reduction: n = round(x) (by adding 1.5 * 2^23, which leaves n
// in the low mantissa bits), f = x - n in [-1/2, 1/2]; 2^f from the degree-3
// minimax polynomial (relative error 7.5e-5) fitted by csrc/fit_exp2.py;
// 2^n applied by adding n to the exponent field.  x is clamped at -126 so
// the exponent add cannot wrap; such terms are below 2^-126 and do not
// matter next to the row maximum (2^0 or more).
__device__ __forceinline__ void ex2_poly2(float &y0, float &y1, float x0,
                                          float x1)
{
    constexpr float kMagic = 12582912.0f; // 1.5 * 2^23
    constexpr float c0 = 9.999280572e-01f, c1 = 6.932609677e-01f,
                    c2 = 2.426111251e-01f, c3 = 5.517166853e-02f;
    x0 = fmaxf(x0, -126.f);
    x1 = fmaxf(x1, -126.f);
    float j0, j1, n0, n1, f0, f1, p0, p1;
    fadd2(j0, j1, x0, x1, kMagic, kMagic);
    fadd2(n0, n1, j0, j1, -kMagic, -kMagic);
    ffma2(f0, f1, n0, n1, -1.f, -1.f, x0, x1);
    ffma2(p0, p1, c3, c3, f0, f1, c2, c2);
    ffma2(p0, p1, p0, p1, f0, f1, c1, c1);
    ffma2(p0, p1, p0, p1, f0, f1, c0, c0);
    y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(j0) << 23));
    y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(j1) << 23));
}

// P (bf16, packed over the S columns) and its row sum for one tile.  With
// EMU, one pair in four is exponentiated by ex2_poly2 and the rest by
// ex2.approx.  A masked entry (score -inf) becomes exactly 0 on the
// special-function unit and 2^-126 on the polynomial path: next to a row sum
// of at least 2^-8 (the row maximum contributes 2^(mt - m_used) >= 2^-8),
// such terms are far below float32 resolution in both l and O.
template <bool EMU>
__device__ __forceinline__ void softmax_p_tile(const float *s, float sl2,
                                               float nm, uint32_t ts,
                                               float *rsum)
{
#pragma unroll
    for (int c4 = 0; c4 < kTcN / 32; ++c4) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
            float x0, x1, x2, x3;
            const int b0 = c4 * 32 + c;
            ffma2(x0, x1, s[b0], s[b0 + 1], sl2, sl2, nm, nm);
            ffma2(x2, x3, s[b0 + 2], s[b0 + 3], sl2, sl2, nm, nm);
            x0 = ex2(x0);
            x1 = ex2(x1);
            if (EMU && ((c >> 2) & 1)) {
                ex2_poly2(x2, x3, x2, x3);
            } else {
                x2 = ex2(x2);
                x3 = ex2(x3);
            }
            const int a = (c >> 2) & 1;
            fadd2(rsum[2 * a], rsum[2 * a + 1], rsum[2 * a], rsum[2 * a + 1], x0, x1);
            fadd2(rsum[2 * a], rsum[2 * a + 1], rsum[2 * a], rsum[2 * a + 1], x2, x3);
            pk[c / 2] = pack_bf16x2(x0, x1);
            pk[c / 2 + 1] = pack_bf16x2(x2, x3);
        }
        tmem_st16(ts + c4 * 16, pk);
    }
}

// Bits [a, b) of a 32-bit word, with a and b clamped to [0, 32].
__device__ __forceinline__ uint32_t range_bits(int a, int b)
{
    a = min(max(a, 0), 32);
    b = min(max(b, 0), 32);
    const uint32_t below_b = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
    const uint32_t below_a = a >= 32 ? 0xffffffffu : ((1u << a) - 1u);
    return below_b & ~below_a;
}

} // namespace bd

namespace bd {

// One key tile of the online softmax for the query row of this thread (its
// TMEM lane), in a warp that holds 32 consecutive rows of a 128-row tile.
//  - S (128 fp32 columns at TMEM address ts) is read into registers.
//  - On a PARTIAL tile, columns outside the row's visible intervals
//    [sp.a0, sp.a1) U [sp.a2, sp.a3), or at or past key khi, become -inf
//    (ks = first key of the tile).
//  - The running maximum m_used (log2 units) is raised lazily, only when the
//    tile maximum exceeds it by more than 8; if any lane raises it and
//    rescale_o is set, the warp waits for the previous PV (wait_prev_pv,
//    false on abort) and rescales its rows of O (128 fp32 columns at t_o) in
//    TMEM.
//  - P = 2^(s * sl2 - m_used) is written as bf16 over S, its sum added to l.
// Returns false if wait_prev_pv failed.  The caller waits for the TMEM
// stores and signals P.
template <bool EMU, typename WaitPV>
__device__ __forceinline__ bool softmax_tile(uint32_t ts, uint32_t t_o, bool full,
                                             const Span &sp, int ks, int khi,
                                             float sl2, bool rescale_o,
                                             float &m_used, float &l,
                                             WaitPV wait_prev_pv)
{
    uint32_t sr[kTcN];
    tmem_ld32x4_wait(ts, ts + 32, ts + 64, ts + 96, sr, sr + 32, sr + 64, sr + 96);
    float s[kTcN];
#pragma unroll
    for (int c = 0; c < kTcN; ++c)
        s[c] = __uint_as_float(sr[c]);
    if (!full) {
        const int e = min(khi, ks + kTcN);
        const int lo0 = max(sp.a0, ks) - ks, hi0 = min(sp.a1, e) - ks;
        const int lo1 = max(sp.a2, ks) - ks, hi1 = min(sp.a3, e) - ks;
#pragma unroll
        for (int w = 0; w < kTcN / 32; ++w) {
            const uint32_t m = range_bits(lo0 - 32 * w, hi0 - 32 * w) |
                               range_bits(lo1 - 32 * w, hi1 - 32 * w);
#pragma unroll
            for (int c = 0; c < 32; ++c)
                s[32 * w + c] = ((m >> c) & 1u) ? s[32 * w + c] : -INFINITY;
        }
    }
    float mc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        mc[i] = fmaxf(s[i], s[8 + i]);
#pragma unroll
    for (int c = 16; c < kTcN; c += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            mc[i] = fmax3(mc[i], s[c + i], s[c + 8 + i]);
    const float mx = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]),
                           fmaxf(mc[6], mc[7]));
    const float mt = mx * sl2;
    // the TMEM read-modify-write of O is warp-collective, so the warp takes
    // it if any lane needs it (with factor 1 on the others)
    const bool need = mt > m_used + 8.f;
    const bool warp_need = __any_sync(0xffffffffu, need);
    float c = 1.f;
    if (need) {
        c = (m_used == -INFINITY) ? 0.f : ex2(m_used - mt);
        l *= c;
        m_used = mt;
    }
    if (rescale_o && warp_need) {
        if (!__all_sync(0xffffffffu, wait_prev_pv()))
            return false;
        tc_fence_after();
#pragma unroll
        for (int q4 = 0; q4 < kTcD / 32; ++q4) {
            uint32_t o[32];
            tmem_ld32_wait(t_o + q4 * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                o[i] = __float_as_uint(__uint_as_float(o[i]) * c);
            tmem_st32(t_o + q4 * 32, o);
        }
    }
    const float nm = (m_used == -INFINITY) ? 0.f : -m_used;
    float rsum[4] = {0.f, 0.f, 0.f, 0.f};
    softmax_p_tile<EMU>(s, sl2, nm, ts, rsum);
    l += (rsum[0] + rsum[1]) + (rsum[2] + rsum[3]);
    return true;
}

} // namespace bd
