// Block-diffusion attention on the 5th-generation tensor cores (sm_100a):
// TMA-staged Q/K/V tiles, tcgen05.mma with fp32 accumulators in tensor
// memory (TMEM), online softmax in registers.
//
// One CTA = one 128-row query tile of one (batch, head) and 6 warps:
//   warps 0-3  softmax warpgroup: thread t owns query row t (TMEM lane t);
//              reads S, masks PARTIAL tiles, keeps the running max / sum,
//              writes P (bf16) back into TMEM over its S buffer, rescales O
//              when the running max grows, and runs the epilogue;
//   warp 4     TMA producer: Q once, then K and V tiles of 128 keys through a
//              kStages-deep shared-memory ring (128-byte swizzle);
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM S
//              buffers, O += P_j V_j with P taken from TMEM; owns the TMEM
//              allocation.
// TMEM (512 columns): S buffer 0 at column 0, S buffer 1 at 128, O at 256.
//
// The visible key set of every row is two intervals (see attn_mma.cuh); the
// key tiles a query tile visits are the union over its rows, and a tile that
// every row sees completely is FULL (no mask work).
//
// Exactness of the lazy rescale: P_j = 2^(x - m_used) where m_used is the
// running maximum the row last rescaled to; it is raised (and O, l rescaled)
// only when the tile maximum exceeds m_used + 8, so P <= 2^8.  out = O / l and
// lse = (m_used + log2 l) ln 2 are exact for any m_used.
//
// Every mbarrier wait is bounded (kWaitCycles); a wait that runs out sets the
// CTA's abort flag and the device status word, after which every role leaves
// its loop, waits (bounded) for its own copies and MMAs in flight, and the
// CTA frees its TMEM and exits.
#pragma once

#include <cuda.h>

#include "attn_mma.cuh"
#include "bd_common.cuh"

namespace bd {

constexpr int kTcThreads = 192;
constexpr int kTcM = 128;     // query rows per CTA
constexpr int kTcN = 128;     // keys per K/V tile
constexpr int kTcD = 128;     // head dim
constexpr int kTcStages = 2;  // K/V ring depth
#ifndef BD_EXP2_EMU
#define BD_EXP2_EMU 1
#endif
// evaluate a quarter of the FULL-tile exponentials with ex2_poly2
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

struct TcParams {
    bf16 *out;
    float *lse;
    float *part_o;
    float *part_lse;
    const int32_t *cache_len;
    int B, Hq, Hkv, L, b;
    int nkeys;   // key rows per kv-head: 2L (fwd) or S_cap (decode)
    int mode;    // decode: 0 bidirectional, 1 causal
    int chunk;   // decode: keys per split
    int nsplit;  // decode
    int qtiles;  // fwd: 128-row query tiles per half
    int rows_unit; // decode: query rows per (batch, kv-head) = group * b
    float scale_log2;
};

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int kSmemQ = 0;
constexpr int kSmemK = kSmemQ + kTileBytes;
constexpr int kSmemV = kSmemK + kTcStages * kTileBytes;
constexpr int kSmemBar = kSmemV + kTcStages * kTileBytes;
constexpr int kTcSmemBytes = kSmemBar + 256 + 1024; // + alignment slack

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

// Bounded wait on phase `parity` of barrier `bar`.  Returns false if the
// CTA was aborted (by this wait running out or by another role).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    for (int it = 0;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 63) == 63) {
            if (*abort_flag)
                return false;
            if (clock64() - t0 > kWaitCycles) {
                *abort_flag = 1;
                raise_device_code(DEV_WAIT_TIMEOUT);
                return false;
            }
        }
    }
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

// 32 lanes x 32 columns of 32-bit TMEM words -> 32 registers per thread
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
          "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
          "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
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
__device__ __forceinline__ void tmem_wait_ld()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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

// P (bf16, packed over the S columns) and its row sum for one tile.  On
// FULL tiles (EMU) one pair in four is exponentiated by ex2_poly2; masked
// entries only occur on the other tiles, where every term goes through
// ex2.approx so that they stay exactly 0.
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

struct TcPlan {
    int nrows;      // valid query rows of the tile
    int row0;       // first query row (fwd: in [0, 2L); decode: local row)
    int qhead;      // TMA 3rd coordinate of Q (fwd: batch*Hq+h; decode: unit)
    int kvhead;     // TMA 3rd coordinate of K/V
    int lo[2], hi[2];
    int flo[2], fhi[2];
    int len, split; // decode
    int gbase;      // decode: global row of local row 0
};

template <int KIND>
__device__ __forceinline__ bool tc_make_plan(const TcParams &p, TcPlan &pl)
{
    if (KIND == 0) {
        const int bh = blockIdx.y;
        const int bi = bh / p.Hq, h = bh % p.Hq;
        const int t = blockIdx.x;
        const int half = t < p.qtiles ? 1 : 0; // clean (heavier) tiles first
        const int idx = p.qtiles - 1 - (t < p.qtiles ? t : t - p.qtiles);
        pl.row0 = (half ? p.L : 0) + idx * kTcM;
        pl.nrows = min(kTcM, p.L - idx * kTcM);
        pl.qhead = bh;
        pl.kvhead = bi * p.Hkv + h / (p.Hq / p.Hkv);
        Span first = fwd_span(p.L, p.b, pl.row0);
        Span last = fwd_span(p.L, p.b, pl.row0 + pl.nrows - 1);
        pl.lo[0] = first.a0; pl.hi[0] = last.a1;
        pl.lo[1] = first.a2; pl.hi[1] = last.a3;
        pl.flo[0] = last.a0; pl.fhi[0] = first.a1;
        pl.flo[1] = last.a2; pl.fhi[1] = first.a3;
        return true;
    } else {
        const int unit = blockIdx.z;
        const int bi = unit / p.Hkv, g = unit % p.Hkv;
        const int group = p.Hq / p.Hkv;
        const int len = p.cache_len[bi];
        const int s = blockIdx.x;
        if (len < 0 || (long long)len + p.b > p.nkeys)
            return false;
        const int total = len + p.b;
        if (s * p.chunk >= total)
            return false;
        pl.len = len;
        pl.split = s;
        pl.row0 = blockIdx.y * kTcM;
        pl.nrows = min(kTcM, p.rows_unit - pl.row0);
        pl.qhead = unit;
        pl.kvhead = unit;
        pl.gbase = (bi * p.Hq + g * group) * p.b;
        const int s0 = s * p.chunk, s1 = min(total, s0 + p.chunk);
        pl.lo[0] = s0; pl.hi[0] = s1;
        pl.lo[1] = 0; pl.hi[1] = 0;
        pl.flo[0] = s0;
        pl.fhi[0] = min(s1, len + (p.mode == 0 ? p.b : 0));
        pl.flo[1] = 0; pl.fhi[1] = 0;
        return true;
    }
}

template <int KIND>
__global__ void __launch_bounds__(kTcThreads, 1)
    bd_tc_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw_addr);

    // barriers
    const uint32_t bar0 = base + kSmemBar;
    const uint32_t bar_q = bar0;                       // Q landed
    auto bar_kfull = [&](int s) { return bar0 + 8 * (1 + s); };
    auto bar_vfull = [&](int s) { return bar0 + 8 * (1 + kTcStages + s); };
    auto bar_kempty = [&](int s) { return bar0 + 8 * (1 + 2 * kTcStages + s); };
    auto bar_vempty = [&](int s) { return bar0 + 8 * (1 + 3 * kTcStages + s); };
    const uint32_t bar_sfull0 = bar0 + 8 * (1 + 4 * kTcStages); // 2 of them
    const uint32_t bar_pfull0 = bar_sfull0 + 16;                // 2 of them
    const uint32_t bar_odone0 = bar_pfull0 + 16;               // 2 of them
    const uint32_t bar_final = bar_odone0 + 16;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + kSmemBar + 200);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sbase + kSmemBar + 208);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    TcPlan pl;
    if (!tc_make_plan<KIND>(p, pl))
        return; // uniform across the CTA

    const int n0 = pl.hi[0] > pl.lo[0] ? (pl.hi[0] - pl.lo[0] + kTcN - 1) / kTcN : 0;
    const int n1 = pl.hi[1] > pl.lo[1] ? (pl.hi[1] - pl.lo[1] + kTcN - 1) / kTcN : 0;
    const int nt = n0 + n1;

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(bar_kfull(s), 1);
            mbar_init(bar_vfull(s), 1);
            mbar_init(bar_kempty(s), 1);
            mbar_init(bar_vempty(s), 1);
        }
        mbar_init(bar_sfull0, 1);
        mbar_init(bar_sfull0 + 8, 1);
        mbar_init(bar_pfull0, 128);
        mbar_init(bar_pfull0 + 8, 128);
        mbar_init(bar_odone0, 1);
        mbar_init(bar_odone0 + 8, 1);
        mbar_init(bar_final, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)), "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) BD_TRACE(7, 0xA110Cu);
    const uint32_t t_s0 = tmem;        // S buffer 0: columns [0, 128)
    const uint32_t t_o = tmem + 256;   // O: columns [256, 384)

    auto tile_of = [&](int it, int &ks, int &rg) {
        rg = it < n0 ? 0 : 1;
        ks = pl.lo[rg] + (it - (rg ? n0 : 0)) * kTcN;
    };

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            mbar_expect_tx(bar_q, kTileBytes);
            tma_load_3d(base + kSmemQ, &tm_q, 0, pl.row0, pl.qhead, bar_q);
            tma_load_3d(base + kSmemQ + kHalfTileBytes, &tm_q, 64, pl.row0,
                        pl.qhead, bar_q);
            int k_issued = 0, v_issued = 0; // tiles whose K / V load was issued
            for (int it = 0; it < nt && ok; ++it) {
                const int s = it % kTcStages;
                const uint32_t ph = ((it / kTcStages) & 1) ^ 1;
                int ks, rg;
                tile_of(it, ks, rg);
                BD_TRACE(1, (it << 4) | 1);
                if (it >= kTcStages && !(ok = mbar_wait(bar_kempty(s), ph, abort_flag)))
                    break;
                BD_TRACE(1, (it << 4) | 2);
                mbar_expect_tx(bar_kfull(s), kTileBytes);
                tma_load_3d(base + kSmemK + s * kTileBytes, &tm_k, 0, ks,
                            pl.kvhead, bar_kfull(s));
                tma_load_3d(base + kSmemK + s * kTileBytes + kHalfTileBytes,
                            &tm_k, 64, ks, pl.kvhead, bar_kfull(s));
                k_issued = it + 1;
                BD_TRACE(1, (it << 4) | 3);
                if (it >= kTcStages && !(ok = mbar_wait(bar_vempty(s), ph, abort_flag)))
                    break;
                BD_TRACE(1, (it << 4) | 4);
                mbar_expect_tx(bar_vfull(s), kTileBytes);
                tma_load_3d(base + kSmemV + s * kTileBytes, &tm_v, 0, ks,
                            pl.kvhead, bar_vfull(s));
                tma_load_3d(base + kSmemV + s * kTileBytes + kHalfTileBytes,
                            &tm_v, 64, ks, pl.kvhead, bar_vfull(s));
                v_issued = it + 1;
            }
            // Wait (bounded) until every copy this role issued has landed, so
            // that no TMA write into shared memory outlives the CTA.
            const long long t0 = clock64();
            auto drain = [&](uint32_t bar, uint32_t par) {
                while (!mbar_try_wait(bar, par) && clock64() - t0 < kWaitCycles) {}
            };
            BD_TRACE(1, 0xD000u | (ok ? 1u : 0u));
            drain(bar_q, 0);
            for (int it = max(0, k_issued - kTcStages); it < k_issued; ++it)
                drain(bar_kfull(it % kTcStages), (it / kTcStages) & 1);
            for (int it = max(0, v_issued - kTcStages); it < v_issued; ++it)
                drain(bar_vfull(it % kTcStages), (it / kTcStages) & 1);
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(kTcM, kTcN, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(kTcM, kTcD, 1);
            bool ok = mbar_wait(bar_q, 0, abort_flag);
            tc_fence_after();
            auto issue_pv = [&](int j) -> bool {
                const int s = j % kTcStages;
                BD_TRACE(0, (j << 4) | 5);
                if (!mbar_wait(bar_pfull0 + 8 * (j & 1), (j >> 1) & 1, abort_flag))
                    return false;
                BD_TRACE(0, (j << 4) | 6);
                if (!mbar_wait(bar_vfull(s), (j / kTcStages) & 1, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t vb = base + kSmemV + s * kTileBytes;
                const uint32_t tp = t_s0 + (j & 1) * 128; // P over S buffer
#pragma unroll
                for (int kk = 0; kk < kTcN / 16; ++kk) {
                    // V is MN-major: 16 keys = two 8-key groups of 1024 B;
                    // the two 64-column halves of d are 16 KB apart.
                    uint64_t bdesc = smem_desc_sw128(vb + kk * 2048,
                                                     kHalfTileBytes, 1024);
                    tc_mma_ts(t_o, tp + kk * 8, bdesc, idesc_pv,
                              (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(bar_odone0 + 8 * (j & 1));
                tc_commit(bar_vempty(s));
                BD_TRACE(0, (j << 4) | 7);
                return true;
            };
            for (int j = 0; j < nt && ok; ++j) {
                const int s = j % kTcStages;
                ok = mbar_wait(bar_kfull(s), (j / kTcStages) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kb = base + kSmemK + s * kTileBytes;
                const uint32_t qb = base + kSmemQ;
                const uint32_t ts = t_s0 + (j & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < kTcD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfTileBytes + (kk & 3) * 32;
                    uint64_t adesc = smem_desc_sw128(qb + off, 16, 1024);
                    uint64_t bdesc = smem_desc_sw128(kb + off, 16, 1024);
                    tc_mma_ss(ts, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar_sfull0 + 8 * (j & 1));
                tc_commit(bar_kempty(s));
                if (j >= 1)
                    ok = issue_pv(j - 1);
            }
            if (ok && nt > 0)
                ok = issue_pv(nt - 1);
            // all MMAs of this CTA retired -> bar_final
            BD_TRACE(0, 0xE000u | (ok ? 1u : 0u));
            tc_commit(bar_final);
            const long long t0 = clock64();
            while (!mbar_try_wait(bar_final, 0) && clock64() - t0 < kWaitCycles) {}
        }
    } else {
        // ------------------------------------------------ softmax warpgroup
        const int row = threadIdx.x; // 0..127 = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const int rl = min(row, pl.nrows - 1);
        Span sp;
        if (KIND == 0) {
            sp = fwd_span(p.L, p.b, pl.row0 + rl);
        } else {
            const int j = (pl.row0 + rl) % p.b;
            const int hi = pl.len + (p.mode == 0 ? p.b : j + 1);
            sp.a0 = pl.split * p.chunk;
            sp.a1 = min(hi, sp.a0 + p.chunk);
            sp.a2 = 0; sp.a3 = 0;
        }
        float m_used = -INFINITY, l = 0.f;
        const float sl2 = p.scale_log2;
        bool ok = true;
        for (int j = 0; j < nt && ok; ++j) {
            int ks, rg;
            tile_of(j, ks, rg);
            const int khi = pl.hi[rg];
            if (lane == 0) BD_TRACE(2 + warp, (j << 4) | 1);
            ok = __all_sync(0xffffffffu,
                            mbar_wait(bar_sfull0 + 8 * (j & 1), (j >> 1) & 1, abort_flag));
            if (!ok) break;
            if (lane == 0) BD_TRACE(2 + warp, (j << 4) | 2);
            tc_fence_after();
            const uint32_t ts = t_s0 + (j & 1) * 128 + lane_off;
            uint32_t sr[128];
            tmem_ld32(ts + 0, sr + 0);
            tmem_ld32(ts + 32, sr + 32);
            tmem_ld32(ts + 64, sr + 64);
            tmem_ld32(ts + 96, sr + 96);
            tmem_wait_ld();
            float s[kTcN];
#pragma unroll
            for (int c = 0; c < kTcN; ++c)
                s[c] = __uint_as_float(sr[c]);
            const bool full = ks >= pl.flo[rg] && ks + kTcN <= pl.fhi[rg] &&
                              ks + kTcN <= khi;
            if (!full) {
                // visible columns of this row inside the tile: two ranges,
                // turned into a 128-bit column mask
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
            // row max: 8 independent chains of three-input max
            float mc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mc[i] = fmaxf(s[i], s[8 + i]);
#pragma unroll
            for (int c = 16; c < kTcN; c += 16)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mc[i] = fmax3(mc[i], s[c + i], s[c + 8 + i]);
            const float mx = fmax3(fmax3(mc[0], mc[1], mc[2]),
                                   fmax3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7]));
            const float mt = mx * sl2; // tile max in the log2 domain
            // Raise m_used only when the tile max exceeds it by more than 8
            // (in log2 units).  The decision is per row, but the TMEM
            // read-modify-write of O is a warp-collective instruction, so the
            // whole warp takes it when any lane needs it (factor 1 elsewhere).
            const bool need = mt > m_used + 8.f;
            const bool warp_need = __any_sync(0xffffffffu, need);
            float c = 1.f;
            if (need) {
                c = (m_used == -INFINITY) ? 0.f : ex2(m_used - mt);
                l *= c;
                m_used = mt;
            }
            if (j >= 1 && warp_need) {
                // O is stable once PV_{j-1} has completed (PV_j needs P_j)
                const int jp = j - 1;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(bar_odone0 + 8 * (jp & 1), (jp >> 1) & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int q4 = 0; q4 < kTcD / 32; ++q4) {
                    uint32_t o[32];
                    tmem_ld32(t_o + lane_off + q4 * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * c);
                    tmem_st32(t_o + lane_off + q4 * 32, o);
                }
            }
            const float nm = (m_used == -INFINITY) ? 0.f : -m_used;
            float rsum[4] = {0.f, 0.f, 0.f, 0.f};
            if (full)
                softmax_p_tile<kEmuExp2>(s, sl2, nm, ts, rsum);
            else
                softmax_p_tile<false>(s, sl2, nm, ts, rsum);
            l += (rsum[0] + rsum[1]) + (rsum[2] + rsum[3]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_pfull0 + 8 * (j & 1));
            if (lane == 0) BD_TRACE(2 + warp, (j << 4) | 3);
        }
        if (ok && nt > 0) {
            const int jl = nt - 1; // PV_{nt-1} done => every PV done
            ok = __all_sync(0xffffffffu,
                            mbar_wait(bar_odone0 + 8 * (jl & 1), (jl >> 1) & 1, abort_flag));
            tc_fence_after();
        }
        // epilogue: O / l -> out, lse
        const bool valid = row < pl.nrows;
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        const float lse_v = (l > 0.f && ok) ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
        if (KIND == 0) {
            const size_t grow = (size_t)pl.qhead * 2 * p.L + pl.row0 + row;
            uint4 *orow = reinterpret_cast<uint4 *>(p.out + grow * kTcD);
#pragma unroll
            for (int q4 = 0; q4 < kTcD / 32; ++q4) {
                uint32_t o[32];
                if (nt > 0 && ok) {
                    tmem_ld32(t_o + lane_off + q4 * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v4;
                        v4.x = pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
                        v4.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                        v4.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                        v4.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                        orow[q4 * 4 + i / 8] = v4;
                    }
                }
            }
            if (valid)
                p.lse[grow] = lse_v;
        } else {
            const size_t rows_all = (size_t)p.B * p.Hq * p.b;
            const size_t grow = (size_t)pl.gbase + pl.row0 + row;
            float4 *orow = reinterpret_cast<float4 *>(
                p.part_o + ((size_t)pl.split * rows_all + grow) * kTcD);
#pragma unroll
            for (int q4 = 0; q4 < kTcD / 32; ++q4) {
                uint32_t o[32];
                if (nt > 0 && ok) {
                    tmem_ld32(t_o + lane_off + q4 * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        orow[q4 * 8 + i / 4] = make_float4(
                            __uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                            __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                }
            }
            if (valid)
                p.part_lse[(size_t)pl.split * rows_all + grow] = lse_v;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) BD_TRACE(6, 0xF00Du);
    if (warp == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

} // namespace bd
