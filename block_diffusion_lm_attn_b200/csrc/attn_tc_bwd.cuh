// Backward of block-diffusion attention, training/prefill form, head dim
// 128, on tcgen05 tensor cores (sm_100a).
//
// Training a block-diffusion LM minimises the BDLM loss ("LLaDA2.0-Uni",
// section "Training objective and loss function", eq. L_BDLM); its gradient
// flows through the attention over [x_t ; x_0] with the three-part block
// mask ("Nemotron-Labs-Diffusion-8B-Base 3x decoding speed-up", section 1).
// Given the forward's out and lse and the upstream gradient dO, for every
// visible (query i, key j) pair of one head:
//     P_ij  = exp(scale q_i.k_j - lse_i)
//     dP_ij = dO_i . v_j,   D_i = dO_i . out_i,   dS_ij = P_ij (dP_ij - D_i)
//     dV_j  = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,
//     dQ_i  = scale sum_j dS_ij k_j
// (q-heads of one GQA group add into their kv-head's dK and dV).
//
// Three kernels, no atomics:
//   bd_bwd_prep_kernel   D_i and lse_i * log2(e) per query row (HBM-bound);
//   bd_bwd_dkdv_kernel   one persistent CTA per SM; a work item is one
//                        128-key tile of one kv-head; it walks the q-heads of
//                        the group and, in 128-row steps, the query rows that
//                        see the tile (the transpose of the forward's key
//                        ranges), accumulating dV and dK in tensor memory;
//   bd_bwd_dq_kernel     one persistent CTA per SM; a work item is one
//                        128-row query tile, walking the forward's key
//                        ranges, accumulating dQ in tensor memory.
// The dQ pass recomputes S and dP (two of the five products) so that no
// partial dQ ever leaves the SM.
#pragma once

#include "attn_tc_persist.cuh"

namespace bd {

struct BParams {
    const bf16 *out, *dout;
    const float *lse;
    float *D;     // [B*Hq*2L] workspace: dO . out
    float *lse2;  // [B*Hq*2L] workspace: lse * log2(e) (+inf for an empty row)
    bf16 *dq, *dk, *dv;
    int B, Hq, Hkv, L, b;
    int qtiles;     // 128-row tiles per half
    int sched_slot; // counter pair of this launch
    int chunk_q;    // dQ: heads per chunk of the work list (as PParams::chunk)
    int chunk_kv;   // dK/dV: (batch, kv-head) groups per chunk of the clean key tiles
    float scale, scale_log2;
};

// ---------------------------------------------------------------------------
// D and lse * log2(e) per query row of 128 values.  A half-warp reduces one
// row from 16-byte loads; each warp takes four rows and issues all its loads
// before any reduction, so enough bytes are in flight to stream at HBM rate.
constexpr int kPrepRowsPerBlock = 32; // 8 warps x 4 rows

__global__ void __launch_bounds__(256)
    bd_bwd_prep_kernel(const BParams p, long long rows)
{
    const int lane = threadIdx.x & 31, hw = lane >> 4, l16 = lane & 15;
    const long long r0 = (long long)blockIdx.x * kPrepRowsPerBlock + (threadIdx.x >> 5) * 4;
    uint4 o[2], g[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const long long r = r0 + 2 * i + hw;
        if (r < rows) {
            o[i] = __ldg(reinterpret_cast<const uint4 *>(p.out + r * kTcD) + l16);
            g[i] = __ldg(reinterpret_cast<const uint4 *>(p.dout + r * kTcD) + l16);
        } else {
            o[i] = make_uint4(0, 0, 0, 0);
            g[i] = o[i];
        }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t ow[4] = {o[i].x, o[i].y, o[i].z, o[i].w};
        const uint32_t gw[4] = {g[i].x, g[i].y, g[i].z, g[i].w};
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            acc = fmaf(__uint_as_float(ow[t] << 16), __uint_as_float(gw[t] << 16), acc);
            acc = fmaf(__uint_as_float(ow[t] & 0xffff0000u), __uint_as_float(gw[t] & 0xffff0000u),
                       acc);
        }
#pragma unroll
        for (int m = 8; m > 0; m >>= 1)
            acc += __shfl_xor_sync(0xffffffffu, acc, m);
        const long long r = r0 + 2 * i + hw;
        if (l16 == 0 && r < rows) {
            p.D[r] = acc;
            const float l = p.lse[r];
            p.lse2[r] = (l == -INFINITY) ? INFINITY : l * kLog2e;
        }
    }
}

// 4-byte global -> shared asynchronous copy; src_bytes = 0 writes zero.
__device__ __forceinline__ void cp_async4(uint32_t dst, const float *src, int src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
// One arrival on `bar` once every cp.async this thread issued so far has
// landed (counted among the barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Stores a warp's 32 rows of 64 bf16 each, held one row per lane (w = the
// row's 32 packed words, lane = row), to row0 + r * stride for r < nvalid.
// Rows written one per lane would make every 16-byte store touch 32
// different lines; instead three xor-shuffle stages transpose the 8 x 8
// grid of 16-byte chunks within each group of eight lanes, after which lane
// 8a + u holds chunk u of rows 8a .. 8a + 7, and each of the eight stores
// writes four whole 128-byte row pieces.
__device__ __forceinline__ void warp_store_rows64(uint32_t (&w)[32], bf16 *row0, size_t stride,
                                                  int nvalid, int lane)
{
    const int u = lane & 7;
#pragma unroll
    for (int m = 4; m >= 1; m >>= 1) {
        const bool hi = (u & m) != 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            if (c & m)
                continue;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t send = hi ? w[4 * c + e] : w[4 * (c | m) + e];
                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
                if (hi)
                    w[4 * c + e] = recv;
                else
                    w[4 * (c | m) + e] = recv;
            }
        }
    }
    const int a = lane >> 3;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int r = 8 * a + k;
        if (r < nvalid)
            reinterpret_cast<uint4 *>(row0 + (size_t)r * stride)[u] =
                make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    }
}

// ---------------------------------------------------------------------------
// Query rows that see key position c (the transpose of fwd_span):
//   noisy key of block k : noisy rows [k b, k b + b)
//   clean key of block k : noisy rows [(k+1) b, L)  U  clean rows [L + k b, 2L)
__device__ __forceinline__ Span key_span(int L, int b, int c)
{
    Span s;
    if (c < L) {
        const int kb = c / b;
        s.a0 = kb * b; s.a1 = kb * b + b; s.a2 = 0; s.a3 = 0;
    } else {
        const int kb = (c - L) / b;
        s.a0 = (kb + 1) * b; s.a1 = L; s.a2 = L + kb * b; s.a3 = 2 * L;
    }
    return s;
}

constexpr int kBwdSub = 128; // query rows per step of the dK/dV kernel
constexpr int kBwdChunkGroups = 8; // (batch, kv-head) groups per chunk of the dK/dV list
static_assert(kBwdSub == 128, "the dK/dV compute warps take 64 query columns each, two per step");

// Work item of the dK/dV kernel: (batch, kv-head) bg and rank r.  Ranks
// 0 .. qtiles-1 are the clean key tiles, idx ascending (heaviest first: a
// clean key tile idx is seen by 2 (qtiles - idx) query tiles of each q-head);
// ranks qtiles .. 2 qtiles-1 the noisy ones (one query tile each).  The list
// holds every clean item first, p.chunk_kv groups at a time (by default
// kBwdChunkGroups) in rank order, so that the running CTAs share the Q and
// dO of a few groups in L2, and then every noisy item.  Group by group, the
// heaviest items of the last groups came near the end of the list: a
// list-scheduling model of the training shape lost 25 % of the pass to its
// tail, against about 1 % this way (an item is up to half of a CTA's average
// load).
struct alignas(16) KvItem {
    int kvhead;       // batch * Hkv + kv-head
    int qhead0;       // batch * Hq + first q-head of the group
    int krow0, nkeys; // first key row (of 2L), valid keys (<= 128)
    int lo0, hi0, lo1, hi1;     // query ranges
    int flo0, fhi0, flo1, fhi1; // queries every key of the tile sees
    int n0, n1;       // steps of range 0 / range 1 per q-head
    int nt;           // steps of the item (all q-heads)
};
static_assert(sizeof(KvItem) <= 64, "a decoded work item takes one 64-byte slot");

__device__ __forceinline__ long long kv_items(const BParams &p)
{
    return (long long)p.B * p.Hkv * 2 * p.qtiles;
}

__device__ __forceinline__ void kv_item(const BParams &p, int w, KvItem &it)
{
    const int NG = p.B * p.Hkv;
    const int nclean = NG * p.qtiles;
    int bg, r;
    if (w < nclean) {
        chunked_rank_order(w, NG, p.qtiles, p.chunk_kv, bg, r);
    } else {
        r = p.qtiles + (w - nclean) / NG;
        bg = (w - nclean) % NG;
    }
    const int clean = r < p.qtiles;
    const int idx = clean ? r : r - p.qtiles;
    const int bi = bg / p.Hkv, g = bg % p.Hkv;
    const int G = p.Hq / p.Hkv;
    it.kvhead = bg;
    it.qhead0 = bi * p.Hq + g * G;
    it.krow0 = (clean ? p.L : 0) + idx * kTcN;
    it.nkeys = min(kTcN, p.L - idx * kTcN);
    const Span first = key_span(p.L, p.b, it.krow0);
    const Span last = key_span(p.L, p.b, it.krow0 + it.nkeys - 1);
    it.lo0 = first.a0; it.hi0 = last.a1;
    it.lo1 = first.a2; it.hi1 = last.a3;
    it.flo0 = last.a0; it.fhi0 = first.a1;
    it.flo1 = last.a2; it.fhi1 = first.a3;
    it.n0 = it.hi0 > it.lo0 ? (it.hi0 - it.lo0 + kBwdSub - 1) / kBwdSub : 0;
    it.n1 = it.hi1 > it.lo1 ? (it.hi1 - it.lo1 + kBwdSub - 1) / kBwdSub : 0;
    it.nt = G * (it.n0 + it.n1);
}

// Step s of an item: q-head s / (n0 + n1), then range 0 or 1.
__device__ __forceinline__ void kv_step(const KvItem &it, int s, int &qhead,
                                        int &qs, int &rg)
{
    const int per = it.n0 + it.n1;
    const int x = s / per, t = s % per;
    qhead = it.qhead0 + x;
    rg = t < it.n0 ? 0 : 1;
    qs = rg == 0 ? it.lo0 + t * kBwdSub : it.lo1 + (t - it.n0) * kBwdSub;
}

// shared memory of the dK/dV kernel
constexpr int kKvStages = 2;
constexpr int kSubBytes = kBwdSub * kTcD * 2;              // one step of Q or dO: 32 KB
constexpr int kKvSmemK = 0;                                // K tile
constexpr int kKvSmemV = kKvSmemK + kTileBytes;            // V tile
constexpr int kKvSmemRing = kKvSmemV + kTileBytes;         // stages: Q, dO
constexpr int kKvStageBytes = 2 * kSubBytes;
constexpr int kKvSmemRows = kKvSmemRing + kKvStages * kKvStageBytes; // lse2, D
constexpr int kKvRowsBytes = 2 * kBwdSub * 4;
constexpr int kKvSmemBar = kKvSmemRows + kKvStages * kKvRowsBytes;
constexpr int kKvSmemSeg = kKvSmemBar + 512; // 4 decoded work items (KvItem)
constexpr int kKvSmemBytes = kKvSmemSeg + 4 * 64 + 1024;
static_assert(kKvStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
static_assert(kKvSmemBytes <= 227 * 1024, "more shared memory than a CTA may have");

// 8 compute warps (two per TMEM lane quarter, each taking half of a row's
// columns), a producer warp and an MMA warp
constexpr int kBwdThreads = 320;
constexpr int kBwdProducerWarp = 8, kBwdMmaWarp = 9;

// Roles: warps 0-7 compute P^T and dS^T (warp w: key rows of TMEM lane
// quarter w & 3, query columns 64 hc .. 64 hc + 63 of each step, hc = w >> 2)
// and write dK, dV out; warp 8 loads (TMA for tiles, cp.async for the
// per-row lse2 and D) and fetches work items; warp 9 issues the MMAs.
// TMEM: dV [0,128), dK [128,256), S^T [256,384), dP^T [384,512); P^T (bf16)
// overwrites the S^T columns of the warp that formed it, dS^T those of dP^T.
// Every product has M = 128 keys and N = 128 (queries or head dim), the
// full-rate shape.  Issue order, step s of 128 query rows:
//   ... dV(s-1), S^T(s), dK(s-1), dP^T(s), dV(s), S^T(s+1), dK(s), ...
// S^T(s+1) rewrites the columns P^T(s) sits in only after dV(s), which reads
// them, was issued, and dP^T(s+1) those of dS^T(s) only after dK(s)
// (tcgen05.mma from one thread execute in issue order).  The compute warps
// form P^T(s) while dK(s-1) and dP^T(s) run, then dS^T(s) (from P^T(s) in
// registers and dP^T(s)) while dV(s) and S^T(s+1) run.
__global__ void __launch_bounds__(kBwdThreads, 1)
    bd_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_qs,
                       const __grid_constant__ CUtensorMap tm_dos,
                       const BParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw_addr);

    const uint32_t bar0 = base + kKvSmemBar;
    const uint32_t bar_kvfull = bar0;        // K and V of the item landed
    const uint32_t bar_kvfree = bar0 + 8;    // every product of the item read K, V
    auto bar_full = [&](int s) { return bar0 + 16 + 8 * s; };                  // stage landed
    auto bar_empty = [&](int s) { return bar0 + 16 + 8 * kKvStages + 8 * s; }; // stage read
    const uint32_t bar1 = bar0 + 16 + 16 * kKvStages;
    const uint32_t bar_sdone = bar1;        // S^T ready
    const uint32_t bar_dpdone = bar1 + 8;   // dP^T ready
    const uint32_t bar_pready = bar1 + 16;  // P^T written
    const uint32_t bar_dsready = bar1 + 24; // dS^T written
    const uint32_t bar_odone = bar1 + 32;   // the item's last dV, dK retired
    const uint32_t bar_ofree = bar1 + 40;   // dV, dK read out
    const uint32_t bar_final = bar1 + 48;
    const uint32_t bar_ifull0 = bar1 + 56;  // 4: work item published
    const uint32_t bar_iempty0 = bar1 + 88; // 4: work item read by all roles
    static_assert(16 + 16 * kKvStages + 120 <= 256, "barriers overlap the item ring");
    volatile int *item_ring = reinterpret_cast<volatile int *>(sbase + kKvSmemBar + 256);
    KvItem *kv_ring = reinterpret_cast<KvItem *>(sbase + kKvSmemSeg);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + kKvSmemBar + 384);
    volatile uint32_t *tmem_slot =
        reinterpret_cast<volatile uint32_t *>(sbase + kKvSmemBar + 392);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar_kvfull, 1);
        mbar_init(bar_kvfree, 1);
        for (int s = 0; s < kKvStages; ++s) {
            mbar_init(bar_full(s), 1 + 32); // expect_tx arrival + one per producer lane
            mbar_init(bar_empty(s), 1);
        }
        mbar_init(bar_sdone, 1);
        mbar_init(bar_dpdone, 1);
        mbar_init(bar_pready, 8); // one arrival per compute warp
        mbar_init(bar_dsready, 8);
        mbar_init(bar_odone, 1);
        mbar_init(bar_ofree, 8);
        mbar_init(bar_final, 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar_ifull0 + 8 * i, 1);
            mbar_init(bar_iempty0 + 8 * i, 257); // MMA + 256 compute threads
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kBwdMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)), "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_dv = tmem, t_dk = tmem + 128, t_st = tmem + 256, t_dp = tmem + 384;

    KvItem it;
    // As in the forward: the producer decodes the item it claims and
    // publishes it in slot si % 4; the other roles copy it (arrive: 0 none,
    // 1 this thread, 2 the converged warp through lane 0).
    auto next_item = [&](int si, bool producer, bool &ok, int arrive = 1) -> bool {
        const int slot = si & 3;
        int w;
        if (producer) {
            if (si >= 4 && !(ok = mbar_wait(bar_iempty0 + 8 * slot,
                                             (uint32_t)(((si - 4) >> 2) & 1), abort_flag)))
                return false;
            if (si == 0)
                sched_claim(p.sched_slot);
            const unsigned int t = atomicAdd(&g_sched_next[p.sched_slot], 1u);
            w = (long long)t < kv_items(p) ? (int)t : -1;
            if (w >= 0) {
                kv_item(p, w, it);
                kv_ring[slot] = it;
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
                it = kv_ring[slot];
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

    if (warp == kBwdProducerWarp) {
        // ------------------------------------------------------ producer
        bool ok = true;
        int si = 0;
        long long g = 0, iss = 0; // running step counter, steps issued
        const long long nrows_all = (long long)p.B * p.Hq * 2 * p.L;
        for (;;) {
            bool got = false;
            if (lane == 0)
                got = next_item(si, true, ok);
            __syncwarp();
            got = __shfl_sync(0xffffffffu, got, 0);
            if (!got)
                break;
            if (lane != 0)
                it = kv_ring[si & 3];
            if (lane == 0) {
                // K, V of item si - 1 are no longer read
                if (si >= 1 && !(ok = mbar_wait(bar_kvfree, (uint32_t)((si - 1) & 1), abort_flag)))
                    got = false;
                if (ok) {
                    mbar_expect_tx(bar_kvfull, 2 * kTileBytes);
                    tma_load_3d(base + kKvSmemK, &tm_k, 0, it.krow0, it.kvhead, bar_kvfull);
                    tma_load_3d(base + kKvSmemK + kHalfTileBytes, &tm_k, 64, it.krow0, it.kvhead,
                                bar_kvfull);
                    tma_load_3d(base + kKvSmemV, &tm_v, 0, it.krow0, it.kvhead, bar_kvfull);
                    tma_load_3d(base + kKvSmemV + kHalfTileBytes, &tm_v, 64, it.krow0, it.kvhead,
                                bar_kvfull);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok)
                break;
            ++si;
            for (int s = 0; s < it.nt && ok; ++s, ++g) {
                const int st = (int)(g % kKvStages);
                int qhead, qs, rg;
                kv_step(it, s, qhead, qs, rg);
                if (lane == 0 && g >= kKvStages)
                    ok = mbar_wait(bar_empty(st), (uint32_t)(((g - kKvStages) / kKvStages) & 1),
                                   abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok)
                    break;
                const uint32_t sb = base + kKvSmemRing + (uint32_t)st * kKvStageBytes;
                if (lane == 0) {
                    mbar_expect_tx(bar_full(st), 2 * kSubBytes);
                    tma_load_3d(sb, &tm_qs, 0, qs, qhead, bar_full(st));
                    tma_load_3d(sb + kSubBytes / 2, &tm_qs, 64, qs, qhead, bar_full(st));
                    tma_load_3d(sb + kSubBytes, &tm_dos, 0, qs, qhead, bar_full(st));
                    tma_load_3d(sb + kSubBytes + kSubBytes / 2, &tm_dos, 64, qs, qhead,
                                bar_full(st));
                    iss = g + 1;
                }
                // lse2 and D of the step's rows, copied asynchronously (so
                // that this warp goes on to the next stage at once); each
                // lane's copies arrive on the stage barrier when they land.
                // Rows outside the range read as 0: the compute warps mask
                // them (a step with such rows is never FULL).
                const int hi = rg == 0 ? it.hi0 : it.hi1;
                const uint32_t sl = base + kKvSmemRows + (uint32_t)st * kKvRowsBytes;
#pragma unroll
                for (int u = 0; u < kBwdSub / 32; ++u) {
                    const int c = lane + 32 * u;
                    const long long row = (long long)qhead * 2 * p.L + qs + c;
                    const bool v = qs + c < hi && row < nrows_all;
                    const long long r0 = v ? row : 0;
                    cp_async4(sl + 4 * c, p.lse2 + r0, v ? 4 : 0);
                    cp_async4(sl + 4 * (kBwdSub + c), p.D + r0, v ? 4 : 0);
                }
                cp_async_arrive_noinc(bar_full(st));
            }
        }
        if (lane == 0) {
            sched_finish(p.sched_slot);
            const long long c0 = clock64();
            auto drain = [&](uint32_t bar, uint32_t par) {
                while (!mbar_try_wait(bar, par) && clock64() - c0 < kWaitCycles) {}
            };
            if (si >= 1)
                drain(bar_kvfull, (uint32_t)((si - 1) & 1));
            for (long long x = iss > kKvStages ? iss - kKvStages : 0; x < iss; ++x)
                drain(bar_full((int)(x % kKvStages)), (uint32_t)((x / kKvStages) & 1));
        }
    } else if (warp == kBwdMmaWarp) {
        // ---------------------------------------------------- MMA issuer
        {
            const uint32_t ld = elect_one();
            constexpr uint32_t idesc_s = idesc_bf16(kTcM, kBwdSub, 0);  // S^T, dP^T
            constexpr uint32_t idesc_g = idesc_bf16(kTcM, kTcD, 1);     // dV, dK
            bool ok = true;
            int si = 0;
            long long g = 0;
            auto stage = [&](long long gg) {
                return base + kKvSmemRing + (uint32_t)(gg % kKvStages) * kKvStageBytes;
            };
            auto wait_stage = [&](long long gg) {
                return mbar_wait_warp(bar_full((int)(gg % kKvStages)),
                                      (uint32_t)((gg / kKvStages) & 1), abort_flag);
            };
            // S^T = K Q^T (A = operand a_tile, B = the stage's Q) or
            // dP^T = V dO^T: M = 128 keys, N = 128 queries, 8 K-steps over d
            auto issue_t = [&](uint32_t acc, uint32_t a_tile, uint32_t b_tile, uint32_t bar) {
#pragma unroll
                for (int kk = 0; kk < kTcD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfTileBytes + (kk & 3) * 32;
                    tc_mma_ss_p(acc, smem_desc_sw128(a_tile + off, 16, 1024),
                                smem_desc_sw128(b_tile + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u,
                                ld);
                }
                tc_commit_p(bar, ld);
            };
            // dV += P^T dO or dK += dS^T Q: A from TMEM (K-step kk = queries
            // 16 kk .. 16 kk + 15, packed by the warps of half kk / 4 at
            // columns 64 (kk / 4) + 8 (kk % 4)), B = dO or Q of the stage
            auto issue_g = [&](uint32_t acc, uint32_t a_tm, uint32_t b_tile, bool first) {
#pragma unroll
                for (int kk = 0; kk < kBwdSub / 16; ++kk) {
                    const uint32_t acol = 64 * (kk >> 2) + 8 * (kk & 3);
                    const uint64_t bd = smem_desc_sw128(b_tile + kk * 2048, kSubBytes / 2, 1024);
                    tc_mma_ts_p(acc, a_tm + acol, bd, idesc_g, (!first || kk > 0) ? 1u : 0u, ld);
                }
            };
            for (;;) {
                const bool got = next_item(si, false, ok, 2);
                ok = __all_sync(0xffffffffu, ok);
                if (!got || !ok)
                    break;
                if (!(ok = mbar_wait_warp(bar_kvfull, (uint32_t)(si & 1), abort_flag)))
                    break;
                if (!(ok = wait_stage(g)))
                    break;
                tc_fence_after();
                issue_t(t_st, base + kKvSmemK, stage(g), bar_sdone);
                issue_t(t_dp, base + kKvSmemV, stage(g) + kSubBytes, bar_dpdone);
                for (int s = 0; s < it.nt && ok; ++s) {
                    const long long gg = g + s;
                    const bool more = s + 1 < it.nt;
                    // dV and dK of the previous item read out
                    if (s == 0 && si >= 1 &&
                        !(ok = mbar_wait_warp(bar_ofree, (uint32_t)((si - 1) & 1), abort_flag)))
                        break;
                    if (!(ok = mbar_wait_warp(bar_pready, (uint32_t)(gg & 1), abort_flag)))
                        break;
                    tc_fence_after();
                    issue_g(t_dv, t_st, stage(gg) + kSubBytes, s == 0);
                    if (more) {
                        if (!(ok = wait_stage(gg + 1)))
                            break;
                        tc_fence_after();
                        issue_t(t_st, base + kKvSmemK, stage(gg + 1), bar_sdone);
                    }
                    if (!(ok = mbar_wait_warp(bar_dsready, (uint32_t)(gg & 1), abort_flag)))
                        break;
                    tc_fence_after();
                    issue_g(t_dk, t_dp, stage(gg), s == 0);
                    tc_commit_p(bar_empty((int)(gg % kKvStages)), ld);
                    if (more)
                        issue_t(t_dp, base + kKvSmemV, stage(gg + 1) + kSubBytes, bar_dpdone);
                }
                if (!ok)
                    break;
                tc_commit_p(bar_kvfree, ld);
                tc_commit_p(bar_odone, ld);
                g += it.nt;
                ++si;
            }
            tc_commit_p(bar_final, ld);
            const long long c0 = clock64();
            while (!mbar_try_wait(bar_final, 0) && clock64() - c0 < kWaitCycles) {}
        }
    } else {
        // ------------------------------------------ P^T, dS^T and epilogue
        // warp w: key rows 32 (w & 3) .. +31 (TMEM lane quarter), query
        // columns 64 hc .. 64 hc + 63 of each step, hc = w >> 2.  The packed
        // P^T / dS^T of half hc go to columns 64 hc .. 64 hc + 31 of the S^T /
        // dP^T buffer: inside the columns this warp itself read, so the other
        // half's loads are never overwritten.
        const int wq = warp & 3, hc = warp >> 2;
        const int row = wq * 32 + lane; // key row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t t_sth = t_st + lane_off + 64 * hc, t_dph = t_dp + lane_off + 64 * hc;
        const float sl2 = p.scale_log2;
        bool ok = true;
        long long g = 0;
        int si = 0;
        for (;;) {
            const bool got = next_item(si, false, ok);
            ok = __all_sync(0xffffffffu, ok);
            if (!got || !ok)
                break;
            const Span ksp = key_span(p.L, p.b, it.krow0 + min(row, it.nkeys - 1));
            for (int s = 0; s < it.nt; ++s) {
                const long long gg = g + s;
                const int st = (int)(gg % kKvStages);
                int qhead, qs, rg;
                kv_step(it, s, qhead, qs, rg);
                // S^T ready; the stage's lse2 / D (written by the producer
                // before its arrival on the stage barrier, which the MMA
                // thread waited for before issuing S^T) landed
                ok = __all_sync(0xffffffffu,
                                mbar_wait(bar_sdone, (uint32_t)(gg & 1), abort_flag) &&
                                    mbar_wait(bar_full(st), (uint32_t)((gg / kKvStages) & 1),
                                              abort_flag));
                if (!ok)
                    break;
                tc_fence_after();
                const float *sl = reinterpret_cast<const float *>(
                                      sbase + kKvSmemRows + st * kKvRowsBytes) + 64 * hc;
                const int hi = rg == 0 ? it.hi0 : it.hi1;
                const int flo = rg == 0 ? it.flo0 : it.flo1;
                const int fhi = rg == 0 ? it.fhi0 : it.fhi1;
                const bool full = qs >= flo && qs + kBwdSub <= fhi && qs + kBwdSub <= hi;
                uint32_t mw[2] = {0xffffffffu, 0xffffffffu};
                if (!full) {
                    const int q0 = qs + 64 * hc;
                    const int e = min(hi, qs + kBwdSub);
                    const int lo0 = max(ksp.a0, q0) - q0, hi0 = min(ksp.a1, e) - q0;
                    const int lo1 = max(ksp.a2, q0) - q0, hi1 = min(ksp.a3, e) - q0;
#pragma unroll
                    for (int w = 0; w < 2; ++w)
                        mw[w] = range_bits(lo0 - 32 * w, hi0 - 32 * w) |
                                range_bits(lo1 - 32 * w, hi1 - 32 * w);
                }
                // P^T = 2^(scale log2(e) s - lse2) over the visible pairs
                float pv[64];
                {
                    uint32_t sr[64], pk[32];
                    tmem_ld32x2_wait(t_sth, t_sth + 32, sr, sr + 32);
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(sl + c);
                        const float la[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int cc = c + u;
                            float xx = fmaf(__uint_as_float(sr[cc]), sl2, -la[u]);
                            if (!((mw[cc >> 5] >> (cc & 31)) & 1u))
                                xx = -INFINITY;
                            pv[cc] = ex2(xx);
                        }
                        pk[c / 2] = pack_bf16x2(pv[c], pv[c + 1]);
                        pk[c / 2 + 1] = pack_bf16x2(pv[c + 2], pv[c + 3]);
                    }
                    tmem_st16(t_sth, pk);
                    tmem_st16(t_sth + 16, pk + 16);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(bar_pready);
                }
                // dS^T = P^T (dP^T - D)
                ok = __all_sync(0xffffffffu, mbar_wait(bar_dpdone, (uint32_t)(gg & 1), abort_flag));
                if (!ok)
                    break;
                tc_fence_after();
                {
                    uint32_t dr[64], dk[32];
                    tmem_ld32x2_wait(t_dph, t_dph + 32, dr, dr + 32);
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        const float4 d4 = *reinterpret_cast<const float4 *>(sl + kBwdSub + c);
                        dk[c / 2] = pack_bf16x2(pv[c] * (__uint_as_float(dr[c]) - d4.x),
                                                pv[c + 1] * (__uint_as_float(dr[c + 1]) - d4.y));
                        dk[c / 2 + 1] = pack_bf16x2(pv[c + 2] * (__uint_as_float(dr[c + 2]) - d4.z),
                                                    pv[c + 3] * (__uint_as_float(dr[c + 3]) - d4.w));
                    }
                    tmem_st16(t_dph, dk);
                    tmem_st16(t_dph + 16, dk + 16);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(bar_dsready);
                }
            }
            if (!ok)
                break;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_odone, (uint32_t)(si & 1), abort_flag));
            if (!ok)
                break;
            tc_fence_after();
            // epilogue: dV and scale * dK, bf16; this thread's row, columns
            // 64 hc .. 64 hc + 63
            const size_t grow0 = (size_t)it.kvhead * 2 * p.L + it.krow0 + wq * 32;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t tb = (which == 0 ? t_dv : t_dk) + lane_off + 64 * hc;
                const float mul = which == 0 ? 1.f : p.scale;
                uint32_t o[64], w[32];
                tmem_ld32x2_wait(tb, tb + 32, o, o + 32);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * mul,
                                       __uint_as_float(o[2 * i + 1]) * mul);
                warp_store_rows64(w, (which == 0 ? p.dv : p.dk) + grow0 * kTcD + 64 * hc, kTcD,
                                  it.nkeys - wq * 32, lane);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_ofree);
            g += it.nt;
            ++si;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

// ---------------------------------------------------------------------------
// dQ: one 128-row query tile per work item, the forward's key ranges.

constexpr int kDqSmemQ = 0;                          // Q tile
constexpr int kDqSmemDO = kDqSmemQ + kTileBytes;     // dO tile
// K and V sit in rings of their own: V(t) is free once dP(t) has run, K(t)
// only after dQ += dS(t) K(t), one tile later, so K gets the deeper ring.
constexpr int kDqKStages = 3;
constexpr int kDqVStages = 2;
constexpr int kDqSmemK = kDqSmemDO + kTileBytes;               // K stages
constexpr int kDqSmemV = kDqSmemK + kDqKStages * kTileBytes;  // V stages
constexpr int kDqSmemBar = kDqSmemV + kDqVStages * kTileBytes;
constexpr int kDqSmemSeg = kDqSmemBar + 512; // 4 decoded work items (Seg)
constexpr int kDqSmemBytes = kDqSmemSeg + 4 * 128 + 1024;
static_assert(sizeof(Seg) <= 128, "a decoded work item takes one 128-byte slot");
static_assert(kDqSmemBytes <= 227 * 1024, "more shared memory than a CTA may have");

// Roles: warps 0-7 compute dS (warp w: query rows of TMEM lane quarter
// w & 3, half w >> 2 of the key columns) and write dQ out; warp 8 loads and
// fetches items; warp 9 issues the MMAs.  TMEM: S [0,128),
// dP [128,256), dQ [256,384), two dS buffers (bf16) [384,448), [448,512).
// Per key tile j: S = Q K^T and dP = dO V^T (after the compute warps have
// read S, dP of tile j - 1 into registers), then dQ += dS(j - 1) K(j - 1).
__global__ void __launch_bounds__(kBwdThreads, 1)
    bd_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const BParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw_addr);

    const uint32_t bar0 = base + kDqSmemBar;
    const uint32_t bar_qfull = bar0;      // Q and dO landed
    const uint32_t bar_qfree = bar0 + 8;  // every S, dP of the item retired
    const uint32_t bar_sfull = bar0 + 16;  // S, dP ready
    const uint32_t bar_sfree = bar0 + 24;  // S, dP read into registers
    auto bar_dsfull = [&](int x) { return bar0 + 32 + 8 * x; };
    auto bar_dsfree = [&](int x) { return bar0 + 48 + 8 * x; };
    const uint32_t bar_qdone = bar0 + 64;  // the item's last dQ retired
    const uint32_t bar_dqfree = bar0 + 72; // dQ read out
    const uint32_t bar_final = bar0 + 80;
    const uint32_t bar_ifull0 = bar0 + 88;
    const uint32_t bar_iempty0 = bar0 + 120;
    auto bar_kfull = [&](int s) { return bar0 + 152 + 8 * s; };
    auto bar_kempty = [&](int s) { return bar0 + 152 + 8 * kDqKStages + 8 * s; };
    auto bar_vfull = [&](int s) { return bar0 + 152 + 16 * kDqKStages + 8 * s; };
    auto bar_vempty = [&](int s) { return bar0 + 152 + 16 * kDqKStages + 8 * kDqVStages + 8 * s; };
    static_assert(152 + 16 * kDqKStages + 16 * kDqVStages <= 256, "barriers overlap the item ring");
    volatile int *item_ring = reinterpret_cast<volatile int *>(sbase + kDqSmemBar + 256);
    Seg *seg_ring = reinterpret_cast<Seg *>(sbase + kDqSmemSeg);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + kDqSmemBar + 384);
    volatile uint32_t *tmem_slot =
        reinterpret_cast<volatile uint32_t *>(sbase + kDqSmemBar + 392);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar_qfull, 1);
        mbar_init(bar_qfree, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_dsfull(s), 8); // one arrival per compute warp
            mbar_init(bar_dsfree(s), 1);
        }
        for (int s = 0; s < kDqKStages; ++s) {
            mbar_init(bar_kfull(s), 1);
            mbar_init(bar_kempty(s), 1);
        }
        for (int s = 0; s < kDqVStages; ++s) {
            mbar_init(bar_vfull(s), 1);
            mbar_init(bar_vempty(s), 1);
        }
        mbar_init(bar_sfull, 1);
        mbar_init(bar_sfree, 8);
        mbar_init(bar_qdone, 1);
        mbar_init(bar_dqfree, 8);
        mbar_init(bar_final, 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar_ifull0 + 8 * i, 1);
            mbar_init(bar_iempty0 + 8 * i, 257); // MMA + 256 compute threads
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kBwdMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)), "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_s = tmem, t_dp = tmem + 128, t_dq = tmem + 256;
    auto t_ds = [&](int x) { return tmem + 384 + 64 * (uint32_t)x; };

    // the forward's work list: (batch * Hq + head, query tile), heaviest first
    PParams fp = {};
    fp.B = p.B; fp.Hq = p.Hq; fp.Hkv = p.Hkv; fp.L = p.L; fp.b = p.b;
    fp.qtiles = p.qtiles;
    fp.chunk = p.chunk_q;
    Seg sg;
    // As in the paired forward: the producer decodes the item it claims and
    // publishes it in slot si % 4; the other roles copy it (arrive: 0 none,
    // 1 this thread, 2 the converged warp through lane 0).
    auto next_item = [&](int si, bool producer, bool &ok, int arrive = 1) -> bool {
        const int slot = si & 3;
        int w;
        if (producer) {
            if (si >= 4 && !(ok = mbar_wait(bar_iempty0 + 8 * slot,
                                             (uint32_t)(((si - 4) >> 2) & 1), abort_flag)))
                return false;
            if (si == 0)
                sched_claim(p.sched_slot);
            const unsigned int t = atomicAdd(&g_sched_next[p.sched_slot], 1u);
            w = (long long)t < FwdSource::items(fp) ? (int)t : -1;
            if (w >= 0) {
                FwdSource::item(fp, w, sg);
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
    auto key_start = [&](int t) {
        return t < sg.n0 ? sg.lo0 + t * kTcN : sg.lo1 + (t - sg.n0) * kTcN;
    };

    if (warp == kBwdProducerWarp) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            bool ok = true;
            int si = 0;
            long long g = 0, issk = 0, issv = 0;
            while (ok && next_item(si, true, ok)) {
                if (si >= 1 && !(ok = mbar_wait(bar_qfree, (uint32_t)((si - 1) & 1), abort_flag)))
                    break;
                mbar_expect_tx(bar_qfull, 2 * kTileBytes);
                tma_load_3d(base + kDqSmemQ, &tm_q, 0, sg.qrow0, sg.qhead, bar_qfull);
                tma_load_3d(base + kDqSmemQ + kHalfTileBytes, &tm_q, 64, sg.qrow0, sg.qhead, bar_qfull);
                tma_load_3d(base + kDqSmemDO, &tm_do, 0, sg.qrow0, sg.qhead, bar_qfull);
                tma_load_3d(base + kDqSmemDO + kHalfTileBytes, &tm_do, 64, sg.qrow0, sg.qhead,
                            bar_qfull);
                ++si;
                for (int t = 0; t < sg.nt; ++t, ++g) {
                    const int ks = key_start(t);
                    const int sk = (int)(g % kDqKStages), sv = (int)(g % kDqVStages);
                    if (g >= kDqKStages &&
                        !(ok = mbar_wait(bar_kempty(sk), (uint32_t)(((g / kDqKStages) - 1) & 1),
                                         abort_flag)))
                        break;
                    const uint32_t kb = base + kDqSmemK + (uint32_t)sk * kTileBytes;
                    mbar_expect_tx(bar_kfull(sk), kTileBytes);
                    tma_load_3d(kb, &tm_k, 0, ks, sg.kvhead, bar_kfull(sk));
                    tma_load_3d(kb + kHalfTileBytes, &tm_k, 64, ks, sg.kvhead, bar_kfull(sk));
                    issk = g + 1;
                    if (g >= kDqVStages &&
                        !(ok = mbar_wait(bar_vempty(sv), (uint32_t)(((g / kDqVStages) - 1) & 1),
                                         abort_flag)))
                        break;
                    const uint32_t vb = base + kDqSmemV + (uint32_t)sv * kTileBytes;
                    mbar_expect_tx(bar_vfull(sv), kTileBytes);
                    tma_load_3d(vb, &tm_v, 0, ks, sg.kvhead, bar_vfull(sv));
                    tma_load_3d(vb + kHalfTileBytes, &tm_v, 64, ks, sg.kvhead, bar_vfull(sv));
                    issv = g + 1;
                }
            }
            sched_finish(p.sched_slot);
            const long long c0 = clock64();
            auto drain = [&](uint32_t bar, uint32_t par) {
                while (!mbar_try_wait(bar, par) && clock64() - c0 < kWaitCycles) {}
            };
            if (si >= 1)
                drain(bar_qfull, (uint32_t)((si - 1) & 1));
            for (long long x = issk > kDqKStages ? issk - kDqKStages : 0; x < issk; ++x)
                drain(bar_kfull((int)(x % kDqKStages)), (uint32_t)((x / kDqKStages) & 1));
            for (long long x = issv > kDqVStages ? issv - kDqVStages : 0; x < issv; ++x)
                drain(bar_vfull((int)(x % kDqVStages)), (uint32_t)((x / kDqVStages) & 1));
        }
    } else if (warp == kBwdMmaWarp) {
        // ---------------------------------------------------- MMA issuer
        {
            const uint32_t ld = elect_one();
            constexpr uint32_t idesc_s = idesc_bf16(kTcM, kTcN, 0);
            constexpr uint32_t idesc_q = idesc_bf16(kTcM, kTcD, 1);
            bool ok = true;
            int si = 0;
            long long j = 0; // running key-tile counter
            // S = Q K^T once K(jg) has landed, dP = dO V^T once V(jg) has;
            // V's stage is free again as soon as dP has run
            auto issue_sdp = [&](long long jg) -> bool {
                const int sk = (int)(jg % kDqKStages), sv = (int)(jg % kDqVStages);
                if (!mbar_wait_warp(bar_kfull(sk), (uint32_t)((jg / kDqKStages) & 1), abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t kb = base + kDqSmemK + (uint32_t)sk * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kTcD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfTileBytes + (kk & 3) * 32;
                    tc_mma_ss_p(t_s, smem_desc_sw128(base + kDqSmemQ + off, 16, 1024),
                                smem_desc_sw128(kb + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u,
                                ld);
                }
                if (!mbar_wait_warp(bar_vfull(sv), (uint32_t)((jg / kDqVStages) & 1), abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t vb = base + kDqSmemV + (uint32_t)sv * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kTcD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfTileBytes + (kk & 3) * 32;
                    tc_mma_ss_p(t_dp, smem_desc_sw128(base + kDqSmemDO + off, 16, 1024),
                                smem_desc_sw128(vb + off, 16, 1024), idesc_s,
                                kk > 0 ? 1u : 0u, ld);
                }
                tc_commit_p(bar_sfull, ld);
                tc_commit_p(bar_vempty(sv), ld);
                return true;
            };
            auto issue_dq = [&](long long jg, bool first) {
                const uint32_t kb = base + kDqSmemK + (uint32_t)(jg % kDqKStages) * kTileBytes;
                const int x = (int)(jg & 1);
#pragma unroll
                for (int kk = 0; kk < kTcN / 16; ++kk) {
                    const uint64_t bk = smem_desc_sw128(kb + kk * 2048, kHalfTileBytes, 1024);
                    tc_mma_ts_p(t_dq, t_ds(x) + kk * 8, bk, idesc_q, (!first || kk > 0) ? 1u : 0u,
                                ld);
                }
                tc_commit_p(bar_dsfree(x), ld);
                tc_commit_p(bar_kempty((int)(jg % kDqKStages)), ld);
            };
            for (;;) {
                const bool got = next_item(si, false, ok, 2);
                ok = __all_sync(0xffffffffu, ok);
                if (!got || !ok)
                    break;
                if (!(ok = mbar_wait_warp(bar_qfull, (uint32_t)(si & 1), abort_flag)))
                    break;
                for (int t = 0; t <= sg.nt && ok; ++t) {
                    const long long jg = j + t;
                    if (t < sg.nt) {
                        // S, dP of the previous tile are in registers
                        if (jg >= 1 && !(ok = mbar_wait_warp(bar_sfree, (uint32_t)((jg - 1) & 1),
                                                             abort_flag)))
                            break;
                        if (!(ok = issue_sdp(jg)))
                            break;
                        if (t == sg.nt - 1)
                            tc_commit_p(bar_qfree, ld);
                    }
                    if (t >= 1) {
                        const long long jp = jg - 1;
                        if (t == 1 && si >= 1 &&
                            !(ok = mbar_wait_warp(bar_dqfree, (uint32_t)((si - 1) & 1),
                                                  abort_flag)))
                            break;
                        if (!(ok = mbar_wait_warp(bar_dsfull((int)(jp & 1)),
                                                  (uint32_t)((jp >> 1) & 1), abort_flag)))
                            break;
                        tc_fence_after();
                        issue_dq(jp, t == 1);
                    }
                }
                if (!ok)
                    break;
                tc_commit_p(bar_qdone, ld);
                j += sg.nt;
                ++si;
            }
            tc_commit_p(bar_final, ld);
            const long long c0 = clock64();
            while (!mbar_try_wait(bar_final, 0) && clock64() - c0 < kWaitCycles) {}
        }
    } else {
        // ---------------------------------------------- dS and epilogue
        // warp w: query rows of TMEM lane quarter w & 3, key columns
        // 64 hc .. 64 hc + 63 of each tile (hc = w >> 2); dS is elementwise,
        // so the two halves of a row need nothing from each other.
        const int wq = warp & 3, hc = warp >> 2;
        const int row = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const float sl2 = p.scale_log2;
        bool ok = true;
        long long j = 0;
        int si = 0;
        for (;;) {
            const bool got = next_item(si, false, ok);
            ok = __all_sync(0xffffffffu, ok);
            if (!got || !ok)
                break;
            const int rl = min(row, sg.nrows - 1);
            const Span sp = fwd_span(p.L, p.b, sg.qrow0 + rl);
            const size_t grow = (size_t)sg.qhead * 2 * p.L + sg.qrow0 + row;
            const bool valid = row < sg.nrows;
            const float lse2 = valid ? p.lse2[grow] : INFINITY;
            const float Dr = valid ? p.D[grow] : 0.f;
            for (int t = 0; t < sg.nt; ++t) {
                const long long jg = j + t;
                const int x = (int)(jg & 1);
                const bool r0 = t < sg.n0;
                const int ks = key_start(t);
                const int khi = r0 ? sg.hi0 : sg.hi1;
                const int flo = r0 ? sg.flo0 : sg.flo1;
                const int fhi = r0 ? sg.fhi0 : sg.fhi1;
                ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull, (uint32_t)(jg & 1), abort_flag));
                if (!ok)
                    break;
                tc_fence_after();
                const bool full = ks >= flo && ks + kTcN <= fhi && ks + kTcN <= khi;
                uint32_t mw[2] = {0xffffffffu, 0xffffffffu};
                if (!full) {
                    const int k0 = ks + 64 * hc;
                    const int e = min(khi, ks + kTcN);
                    const int lo0 = max(sp.a0, k0) - k0, hi0 = min(sp.a1, e) - k0;
                    const int lo1 = max(sp.a2, k0) - k0, hi1 = min(sp.a3, e) - k0;
#pragma unroll
                    for (int w = 0; w < 2; ++w)
                        mw[w] = range_bits(lo0 - 32 * w, hi0 - 32 * w) |
                                range_bits(lo1 - 32 * w, hi1 - 32 * w);
                }
                uint32_t sr[64], dr[64], pk[32];
                tmem_ld32x4_wait(t_s + lane_off + 64 * hc, t_s + lane_off + 64 * hc + 32,
                                 t_dp + lane_off + 64 * hc, t_dp + lane_off + 64 * hc + 32, sr,
                                 sr + 32, dr, dr + 32);
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar_sfree); // S, dP may be overwritten
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    float x0 = fmaf(__uint_as_float(sr[c]), sl2, -lse2);
                    float x1 = fmaf(__uint_as_float(sr[c + 1]), sl2, -lse2);
                    if (!((mw[c >> 5] >> (c & 31)) & 1u))
                        x0 = -INFINITY;
                    if (!((mw[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u))
                        x1 = -INFINITY;
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    pk[c / 2] = pack_bf16x2(p0 * (__uint_as_float(dr[c]) - Dr),
                                            p1 * (__uint_as_float(dr[c + 1]) - Dr));
                }
                // dS buffer x was last read by dQ of tile jg - 2 (issued
                // while this warp worked on tile jg - 1)
                if (jg >= 2) {
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_dsfree(x), (uint32_t)(((jg - 2) >> 1) & 1),
                                                           abort_flag));
                    if (!ok)
                        break;
                    tc_fence_after();
                }
                tmem_st16(t_ds(x) + lane_off + 32 * hc, pk);
                tmem_st16(t_ds(x) + lane_off + 32 * hc + 16, pk + 16);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar_dsfull(x));
            }
            if (!ok)
                break;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_qdone, (uint32_t)(si & 1), abort_flag));
            if (!ok)
                break;
            tc_fence_after();
            // the warp's 32 rows, dQ columns 64 hc .. 64 hc + 63
            {
                uint32_t o[64], w[32];
                tmem_ld32x2_wait(t_dq + lane_off + 64 * hc, t_dq + lane_off + 64 * hc + 32, o,
                                 o + 32);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * p.scale,
                                       __uint_as_float(o[2 * i + 1]) * p.scale);
                warp_store_rows64(w, p.dq + (grow - lane) * kTcD + 64 * hc, kTcD,
                                  sg.nrows - wq * 32, lane);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_dqfree);
            j += sg.nt;
            ++si;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

} // namespace bd
