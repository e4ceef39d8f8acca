// Persistent tcgen05 block-diffusion attention, training/prefill form, two
// query tiles per CTA.
//
// A work item is one 128-row query tile of two query heads that read the
// same kv-head (heads 2i and 2i + 1 of a GQA group): their key ranges and
// masks are identical, so every K/V tile brought into shared memory serves
// 256 query rows.  Two softmax warpgroups, one per query tile, alternate on
// the tensor pipe: while one computes P from its S, the tensor cores run the
// other's PV and next QK, so each MMA wait covers twice the work of the
// one-tile kernel and K/V traffic from L2 halves.
//
// Roles: warps 0-3 softmax and epilogue of tile A (thread t = row t = TMEM
// lane t), warps 4-7 the same for tile B, warp 8 TMA producer of Q and K
// (and the work-item fetch), warp 9 MMA issuer, warp 10 TMA producer of V,
// warp 11 idle.  All 32 lanes of warp 9 run the issue loop and its barrier
// waits; one elected lane issues each tcgen05.mma and tcgen05.commit as a
// predicated instruction.  (An issue loop run by one lane inside a divergent
// branch measured about 50 cycles per MMA and per commit on the issuing side,
// against about 19 and 3 this way, and the tensor pipe idled between
// groups.)  setmaxnreg moves registers from warpgroup 2 to the two
// softmax warpgroups.
//
// TMEM: S_A columns [0, 128), S_B [128, 256), O_A [256, 384), O_B [384, 512);
// P (bf16) overwrites its own S.  Shared memory: the two Q tiles of the
// current item (one buffer), two K and two V stages, per-warp output
// staging, barriers.
//
// MMA issue order per key tile j (the chains of A and B interleave):
//   PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1)
// so QK_A(j+1) overwrites S_A only after PV_A(j) -- which read P_A(j) from
// it -- was issued (tcgen05.mma from one thread execute in issue order).
#pragma once

#include "attn_tc_persist.cuh"

namespace bd {

constexpr int kPairThreads = 384;
// query tiles per half from which the paired kernel runs its EMU variant:
// measured on B200, the training shape (16 tiles, items of ~9 key tiles) 3 %
// faster with, the long context (64 tiles, ~32 key tiles) 1.4 % faster with.
// (Before each item was decoded once, in the producer, the training shape
// was 1.5 % faster without: the extra instructions then landed on the item
// boundaries' critical path.)
constexpr int kPairEmuQtiles = 16;
constexpr int kPairRegsSoftmax = 208; // setmaxnreg of warpgroups 0 and 1
constexpr int kPairRegsOther = 88;    // setmaxnreg of warpgroup 2
static_assert(2 * 128 * kPairRegsSoftmax + 128 * kPairRegsOther <=
                  kPairThreads * (65536 / kPairThreads / 8 * 8),
              "register split above the launch's allocation");

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int kPairSmemQ = 0;                           // tiles A, B
constexpr int kPairSmemK = kPairSmemQ + 2 * kTileBytes; // 2 stages
constexpr int kPairSmemV = kPairSmemK + 2 * kTileBytes; // 2 stages
constexpr int kPairSmemEpi = kPairSmemV + 2 * kTileBytes; // 8 warps x 4 KB
constexpr int kPairSmemBar = kPairSmemEpi + 8 * 32 * 128;
constexpr int kPairSmemSeg = kPairSmemBar + 512; // 4 decoded work items (PairSeg)
constexpr int kPairSmemBytes = kPairSmemSeg + 4 * 64 + 1024;
static_assert(kPairSmemBytes <= 227 * 1024, "more shared memory than a CTA may have");

// Work item w of the pair kernel: (batch, head pair) bp and cost rank r
// (0 = heaviest) in chunked rank order, as FwdSource with head pairs for heads.
struct alignas(16) PairSeg {
    int qhead;  // global index (batch * Hq + head) of tile A; tile B is +1
    int qrow0, nrows, kvhead;
    int lo0, hi0, lo1, hi1;
    int flo0, fhi0, flo1, fhi1;
    int n0, nt;
};
static_assert(sizeof(PairSeg) <= 64, "a decoded work item takes one 64-byte slot");

__device__ __forceinline__ long long pair_items(const PParams &p)
{
    return (long long)p.B * (p.Hq / 2) * 2 * p.qtiles;
}

__device__ __forceinline__ void pair_item(const PParams &p, int w, PairSeg &sg)
{
    const int R = 2 * p.qtiles;
    int bp, r; // bp = batch * (Hq / 2) + pair
    chunked_rank_order(w, p.B * (p.Hq / 2), R, p.chunk, bp, r);
    const int idx = p.qtiles - 1 - (r >> 1);
    const int clean = r & 1;
    const int half = p.Hq / 2;
    const int bi = bp / half, pi = bp % half;
    sg.qrow0 = (clean ? p.L : 0) + idx * kTcM;
    sg.nrows = min(kTcM, p.L - idx * kTcM);
    sg.qhead = bi * p.Hq + 2 * pi;
    sg.kvhead = bi * p.Hkv + (2 * pi) / (p.Hq / p.Hkv);
    const Span first = fwd_span(p.L, p.b, sg.qrow0);
    const Span last = fwd_span(p.L, p.b, sg.qrow0 + sg.nrows - 1);
    sg.lo0 = first.a0; sg.hi0 = last.a1;
    sg.lo1 = first.a2; sg.hi1 = last.a3;
    sg.flo0 = last.a0; sg.fhi0 = first.a1;
    sg.flo1 = last.a2; sg.fhi1 = first.a3;
    sg.n0 = sg.hi0 > sg.lo0 ? (sg.hi0 - sg.lo0 + kTcN - 1) / kTcN : 0;
    const int n1 = sg.hi1 > sg.lo1 ? (sg.hi1 - sg.lo1 + kTcN - 1) / kTcN : 0;
    sg.nt = sg.n0 + n1;
}

// DH: head dim of the tensors, 128, or 64 / 32 read zero-extended to 128
// columns (the QKs skip the zero K-steps; the columns of O past DH are never
// written).  EMU: a quarter of each tile's exponentials on the FMA pipe
// (ex2_poly2).  That pays on long work items, where the softmax runs in
// steady state, and costs on short ones, where the extra instructions land
// on the item boundaries' critical path; the launch chooses (kPairEmuQtiles).
template <int DH, bool EMU>
__global__ void __launch_bounds__(kPairThreads, 1)
    bd_tc_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw_addr);

    const uint32_t bar0 = base + kPairSmemBar;
    const uint32_t bar_qfull = bar0;          // both Q tiles landed
    const uint32_t bar_qfree = bar0 + 8;      // every QK of the item retired
    auto bar_kfull = [&](int s) { return bar0 + 16 + 8 * s; };
    auto bar_vfull = [&](int s) { return bar0 + 32 + 8 * s; };
    auto bar_kempty = [&](int s) { return bar0 + 48 + 8 * s; };
    auto bar_vempty = [&](int s) { return bar0 + 64 + 8 * s; };
    auto bar_sfull = [&](int x) { return bar0 + 80 + 8 * x; };  // S_x ready
    auto bar_pfull = [&](int x) { return bar0 + 96 + 8 * x; };  // P_x written
    auto bar_odone = [&](int x, int par) { return bar0 + 112 + 16 * x + 8 * par; };
    auto bar_ofree = [&](int x) { return bar0 + 144 + 8 * x; }; // O_x read out
    const uint32_t bar_final = bar0 + 160;
    const uint32_t bar_ifull0 = bar0 + 168;  // 4: work item published
    const uint32_t bar_iempty0 = bar0 + 200; // 4: work item read by all roles
    volatile int *item_ring = reinterpret_cast<volatile int *>(sbase + kPairSmemBar + 256);
    PairSeg *seg_ring = reinterpret_cast<PairSeg *>(sbase + kPairSmemSeg);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + kPairSmemBar + 384);
    volatile uint32_t *tmem_slot =
        reinterpret_cast<volatile uint32_t *>(sbase + kPairSmemBar + 392);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(bar_qfull, 1);
        mbar_init(bar_qfree, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_kfull(s), 1);
            mbar_init(bar_vfull(s), 1);
            mbar_init(bar_kempty(s), 1);
            mbar_init(bar_vempty(s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar_sfull(x), 1);
            mbar_init(bar_pfull(x), 128);
            mbar_init(bar_odone(x, 0), 1);
            mbar_init(bar_odone(x, 1), 1);
            mbar_init(bar_ofree(x), 128);
        }
        mbar_init(bar_final, 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar_ifull0 + 8 * i, 1);
            mbar_init(bar_iempty0 + 8 * i, 258); // MMA, V producer, 256 softmax threads
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 9) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)), "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    PairSeg sg;
    // Next item of this CTA, identical for every role: the Q/K producer
    // takes it from the launch's global counter, decodes it (pair_item, a
    // few integer divisions: ~1800 cycles of one warp, measured) and
    // publishes index and decoded item in slot si % 4; the other roles copy
    // the decoded item, so the divisions stay off the softmax and MMA paths.
    // arrive: 0 none, 1 this thread, 2 the whole (converged) warp, through
    // lane 0 once every lane has read the slot.
    auto next_seg = [&](int si, bool producer, bool &ok, int arrive = 1) -> bool {
        const int slot = si & 3;
        int w;
        if (producer) {
            if (si >= 4 && !(ok = mbar_wait(bar_iempty0 + 8 * slot,
                                             (uint32_t)(((si - 4) >> 2) & 1), abort_flag)))
                return false;
            if (si == 0)
                sched_claim(p.sched_slot);
            const unsigned int t = atomicAdd(&g_sched_next[p.sched_slot], 1u);
            w = (long long)t < pair_items(p) ? (int)t : -1;
            if (w >= 0) {
                pair_item(p, w, sg);
                seg_ring[slot] = sg;
            }
            item_ring[slot] = w;
            mbar_arrive(bar_ifull0 + 8 * slot);
        } else {
            ok = mbar_wait(bar_ifull0 + 8 * slot, (uint32_t)((si >> 2) & 1), abort_flag);
            if (arrive == 2) // one outcome for the warp before its __syncwarp
                ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                return false;
            w = item_ring[slot];
            if (w >= 0)
                sg = seg_ring[slot];
            if (arrive == 2) {
                __syncwarp();
                if ((threadIdx.x & 31) == 0)
                    mbar_arrive(bar_iempty0 + 8 * slot);
            } else if (arrive == 1) {
                mbar_arrive(bar_iempty0 + 8 * slot);
            }
        }
        return w >= 0;
    };
    auto key_start = [&](int it) {
        return it < sg.n0 ? sg.lo0 + it * kTcN : sg.lo1 + (it - sg.n0) * kTcN;
    };

    if (warp >= 8) {
    // warpgroup 2 gives registers to the softmax warpgroups; every warp of
    // it executes this one instruction
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairRegsOther));
    if (warp == 8) {
        // ---------------------------------------- TMA producer: Q and K
        if (lane == 0) {
            bool ok = true;
            int si = 0;
            long long g = 0, kiss = 0;
            while (ok && next_seg(si, true, ok)) {
                // the Q buffer was last read by the QKs of item si - 1
                if (si >= 1 && !(ok = mbar_wait(bar_qfree, (uint32_t)((si - 1) & 1), abort_flag)))
                    break;
                mbar_expect_tx(bar_qfull, 2 * kTileBytes);
                for (int x = 0; x < 2; ++x) {
                    const uint32_t dst = base + kPairSmemQ + (uint32_t)x * kTileBytes;
                    tma_load_3d(dst, &tm_q, 0, sg.qrow0, sg.qhead + x, bar_qfull);
                    tma_load_3d(dst + kHalfTileBytes, &tm_q, 64, sg.qrow0, sg.qhead + x,
                                bar_qfull);
                }
                ++si;
                for (int it = 0; it < sg.nt; ++it, ++g) {
                    const int s = (int)(g & 1);
                    // stage s was last read by QK_A and QK_B of tile g - 2
                    if (g >= 2 && !(ok = mbar_wait(bar_kempty(s),
                                                   (uint32_t)((g >> 1) & 1) ^ 1u, abort_flag)))
                        break;
                    if (g == 0 && blockIdx.x == 0 && atomicExch(&g_fault_skip_k, 0) != 0)
                        continue; // injected fault: this tile never arrives
                    const int ks = key_start(it);
                    mbar_expect_tx(bar_kfull(s), kTileBytes);
                    tma_load_3d(base + kPairSmemK + s * kTileBytes, &tm_k, 0, ks, sg.kvhead,
                                bar_kfull(s));
                    tma_load_3d(base + kPairSmemK + s * kTileBytes + kHalfTileBytes, &tm_k, 64,
                                ks, sg.kvhead, bar_kfull(s));
                    kiss = g + 1;
                }
            }
            // this CTA takes no more items; the last CTA resets the pair
            sched_finish(p.sched_slot);
            // wait (bounded) for every copy this role issued
            const long long c0 = clock64();
            auto drain = [&](uint32_t bar, uint32_t par) {
                while (!mbar_try_wait(bar, par) && clock64() - c0 < kWaitCycles) {}
            };
            if (si >= 1)
                drain(bar_qfull, (uint32_t)((si - 1) & 1));
            for (long long x = kiss > 2 ? kiss - 2 : 0; x < kiss; ++x)
                drain(bar_kfull((int)(x & 1)), (uint32_t)((x >> 1) & 1));
        }
    } else if (warp == 10) {
        // ---------------------------------------------- TMA producer: V
        if (lane == 0) {
            bool ok = true;
            int si = 0;
            long long g = 0, viss = 0;
            while (ok && next_seg(si, false, ok)) {
                ++si;
                for (int it = 0; it < sg.nt; ++it, ++g) {
                    const int s = (int)(g & 1);
                    // stage s was last read by PV_A and PV_B of tile g - 2
                    if (g >= 2 && !(ok = mbar_wait(bar_vempty(s),
                                                   (uint32_t)((g >> 1) & 1) ^ 1u, abort_flag)))
                        break;
                    const int ks = key_start(it);
                    mbar_expect_tx(bar_vfull(s), kTileBytes);
                    tma_load_3d(base + kPairSmemV + s * kTileBytes, &tm_v, 0, ks, sg.kvhead,
                                bar_vfull(s));
                    tma_load_3d(base + kPairSmemV + s * kTileBytes + kHalfTileBytes, &tm_v, 64,
                                ks, sg.kvhead, bar_vfull(s));
                    viss = g + 1;
                }
            }
            const long long c0 = clock64();
            for (long long x = viss > 2 ? viss - 2 : 0; x < viss; ++x)
                while (!mbar_try_wait(bar_vfull((int)(x & 1)), (uint32_t)((x >> 1) & 1)) &&
                       clock64() - c0 < kWaitCycles) {}
        }
    } else if (warp == 9) {
        // ---------------------------------------------------- MMA issuer
        // The whole warp runs the loop (waits, bookkeeping); the MMAs and
        // commits are issued by the elected lane as predicated instructions.
        {
            const uint32_t ld = elect_one();
            constexpr uint32_t idesc_qk = idesc_bf16(kTcM, kTcN, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(kTcM, kTcD, 1);
            bool ok = true;
            int si = 0;
            long long j = 0; // running key-tile counter
            auto issue_qk = [&](int x, long long jg) {
                const uint32_t kb = base + kPairSmemK + (uint32_t)(jg & 1) * kTileBytes;
                const uint32_t qb = base + kPairSmemQ + (uint32_t)x * kTileBytes;
                const uint32_t ts = tmem + (uint32_t)x * 128;
#pragma unroll
                for (int kk = 0; kk < kTcD / 16; ++kk) {
                    if (kk * 16 >= DH) // zero columns of a head dim below 128
                        break;
                    const uint32_t off = (kk >> 2) * kHalfTileBytes + (kk & 3) * 32;
                    tc_mma_ss_p(ts, smem_desc_sw128(qb + off, 16, 1024),
                                smem_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u,
                                ld);
                }
                tc_commit_p(bar_sfull(x), ld);
            };
            auto issue_pv = [&](int x, long long jg, bool first) {
                const uint32_t vb = base + kPairSmemV + (uint32_t)(jg & 1) * kTileBytes;
                const uint32_t tp = tmem + (uint32_t)x * 128;
                const uint32_t to = tmem + 256 + (uint32_t)x * 128;
#pragma unroll
                for (int kk = 0; kk < kTcN / 16; ++kk) {
                    uint64_t bdesc = smem_desc_sw128(vb + kk * 2048, kHalfTileBytes, 1024);
                    tc_mma_ts_p(to, tp + kk * 8, bdesc, idesc_pv, (!first || kk > 0) ? 1u : 0u, ld);
                }
                tc_commit_p(bar_odone(x, (int)(jg & 1)), ld);
            };
            auto wait_k = [&](long long jg) {
                return mbar_wait_warp(bar_kfull((int)(jg & 1)), (uint32_t)((jg >> 1) & 1),
                                      abort_flag);
            };
            for (;;) {
                const bool got = next_seg(si, false, ok, 2);
                ok = __all_sync(0xffffffffu, ok);
                if (!got || !ok)
                    break;
                if (!(ok = mbar_wait_warp(bar_qfull, (uint32_t)(si & 1), abort_flag)))
                    break;
                if (!(ok = wait_k(j)))
                    break;
                tc_fence_after();
                issue_qk(0, j);
                issue_qk(1, j);
                tc_commit_p(bar_kempty((int)(j & 1)), ld);
                if (sg.nt == 1)
                    tc_commit_p(bar_qfree, ld);
                for (int jj = 0; jj < sg.nt && ok; ++jj) {
                    const long long jg = j + jj;
                    const bool more = jj + 1 < sg.nt;
                    // PV_A(jg), then QK_A(jg + 1) into S_A
                    if (jj == 0 && si >= 1 &&
                        !(ok = mbar_wait_warp(bar_ofree(0), (uint32_t)((si - 1) & 1), abort_flag)))
                        break;
                    if (!(ok = mbar_wait_warp(bar_pfull(0), (uint32_t)(jg & 1), abort_flag)))
                        break;
                    if (!(ok = mbar_wait_warp(bar_vfull((int)(jg & 1)), (uint32_t)((jg >> 1) & 1),
                                              abort_flag)))
                        break;
                    tc_fence_after();
                    issue_pv(0, jg, jj == 0);
                    if (more) {
                        if (!(ok = wait_k(jg + 1)))
                            break;
                        tc_fence_after();
                        issue_qk(0, jg + 1);
                    }
                    // PV_B(jg), then QK_B(jg + 1) into S_B
                    if (jj == 0 && si >= 1 &&
                        !(ok = mbar_wait_warp(bar_ofree(1), (uint32_t)((si - 1) & 1), abort_flag)))
                        break;
                    if (!(ok = mbar_wait_warp(bar_pfull(1), (uint32_t)(jg & 1), abort_flag)))
                        break;
                    tc_fence_after();
                    issue_pv(1, jg, jj == 0);
                    tc_commit_p(bar_vempty((int)(jg & 1)), ld);
                    if (more) {
                        issue_qk(1, jg + 1);
                        tc_commit_p(bar_kempty((int)((jg + 1) & 1)), ld);
                        if (jj + 2 == sg.nt)
                            tc_commit_p(bar_qfree, ld);
                    }
                }
                if (!ok)
                    break;
                j += sg.nt;
                ++si;
            }
            tc_commit_p(bar_final, ld);
            const long long c0 = clock64();
            while (!mbar_try_wait(bar_final, 0) && clock64() - c0 < kWaitCycles) {}
        }
    }
    } else {
        // -------------------------------------------- softmax + epilogue
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPairRegsSoftmax));
        const int x = warp >> 2;          // 0: tile A, 1: tile B
        const int wq = warp & 3;          // TMEM lane quarter
        const int row = threadIdx.x & 127;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t t_s = tmem + (uint32_t)x * 128;
        const uint32_t t_o = tmem + 256 + (uint32_t)x * 128;
        const float sl2 = p.scale_log2;
        bool ok = true;
        long long j = 0;
        int si = 0;
        for (;;) {
            const bool got = next_seg(si, false, ok);
            ok = __all_sync(0xffffffffu, ok);
            if (!got || !ok)
                break;
            const int rl = min(row, sg.nrows - 1);
            const Span sp = fwd_span(p.L, p.b, sg.qrow0 + rl);
            float m_used = -INFINITY, l = 0.f;
            for (int jj = 0; jj < sg.nt; ++jj) {
                const long long jg = j + jj;
                const bool r0 = jj < sg.n0;
                const int ks = key_start(jj);
                const int khi = r0 ? sg.hi0 : sg.hi1;
                const int flo = r0 ? sg.flo0 : sg.flo1;
                const int fhi = r0 ? sg.fhi0 : sg.fhi1;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(bar_sfull(x), (uint32_t)(jg & 1), abort_flag));
                if (!ok)
                    break;
                tc_fence_after();
                const bool full = ks >= flo && ks + kTcN <= fhi && ks + kTcN <= khi;
                const long long jp = jg - 1;
                ok = softmax_tile<EMU>(
                    t_s + lane_off, t_o + lane_off, full, sp, ks, khi, sl2, jj >= 1, m_used, l,
                    [&] {
                        return mbar_wait(bar_odone(x, (int)(jp & 1)), (uint32_t)((jp >> 1) & 1),
                                         abort_flag);
                    });
                if (!ok)
                    break;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_pfull(x));
            }
            if (!ok)
                break;
            {
                const long long jl = j + sg.nt - 1; // last PV of the item
                ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(x, (int)(jl & 1)),
                                                       (uint32_t)((jl >> 1) & 1), abort_flag));
                if (!ok)
                    break;
                tc_fence_after();
            }
            // ------------------------------------------------ epilogue
            // Rows go out through this warp's 4 KB staging area, one
            // 64-column half at a time, so that each global store writes four
            // 128-byte row pieces instead of 16-byte pieces of 32 rows.  Chunk
            // c (16 bytes) of row l sits at l * 128 + ((c ^ (l & 7)) << 4).
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            const float lse_v = (l > 0.f) ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
            const size_t head_row0 = (size_t)(sg.qhead + x) * 2 * p.L + sg.qrow0;
            const uint32_t epi = base + kPairSmemEpi + (uint32_t)warp * (32 * 128);
            // O in one load (one TMEM round trip, not one per 32 columns);
            // once it is in registers the next item's first PV may overwrite it
            uint32_t ov[kTcD];
            if constexpr (DH > 64)
                tmem_ld32x4_wait(t_o + lane_off, t_o + lane_off + 32, t_o + lane_off + 64,
                                 t_o + lane_off + 96, ov, ov + 32, ov + 64, ov + 96);
            else if constexpr (DH > 32)
                tmem_ld32x2_wait(t_o + lane_off, t_o + lane_off + 32, ov, ov + 32);
            else
                tmem_ld32_wait(t_o + lane_off, ov);
            tc_fence_before();
            mbar_arrive(bar_ofree(x));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h * 64 >= DH) // O columns past the head dim are not output
                    break;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int q4 = 2 * h + q;
                    if (q4 * 32 >= DH)
                        break;
                    const uint32_t *o = ov + q4 * 32;
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        const uint32_t cch = (uint32_t)(q * 4 + i / 8);
                        const uint32_t a = epi + (uint32_t)lane * 128 +
                                           ((cch ^ (uint32_t)(lane & 7)) << 4);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                                     "r"(pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv)),
                                     "r"(pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv)),
                                     "r"(pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv)),
                                     "r"(pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv))
                                     : "memory");
                    }
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 4 * i + (lane >> 3); // row within the warp's 32
                    const uint32_t cc = (uint32_t)(lane & 7);
                    uint32_t x0, x1, x2, x3;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
                                 : "r"(epi + (uint32_t)r * 128 + ((cc ^ (uint32_t)(r & 7)) << 4))
                                 : "memory");
                    const int trow = wq * 32 + r;
                    if (trow < sg.nrows && h * 64 + (int)cc * 8 < DH)
                        reinterpret_cast<uint4 *>(p.out + (head_row0 + trow) * DH)[h * 8 + cc] =
                            make_uint4(x0, x1, x2, x3);
                }
                __syncwarp();
            }
            if (row < sg.nrows)
                p.lse[head_row0 + row] = lse_v;
            j += sg.nt;
            ++si;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

} // namespace bd
