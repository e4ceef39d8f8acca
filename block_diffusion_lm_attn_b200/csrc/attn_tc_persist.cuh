// Persistent tcgen05 block-diffusion attention kernel, shared by the
// training/prefill form and the block-decode form.
//
// The grid is one CTA per SM.  Each CTA walks a list of SEGMENTS; a segment
// is one 128-row query tile and a run of 128-key K/V tiles:
//   training/prefill: every (batch, head, query tile) is one work item,
//     handed out dynamically from a global counter, heaviest first across a
//     few heads at a time (see FwdSource);
//   block decode: the (unit, key tile) space -- a unit is one (sequence,
//     kv-head, 128-row query tile) -- is cut into G equal contiguous ranges
//     (stream-K), or, when the units are few and balanced, dealt one unit
//     per CTA.  A unit that lies inside one CTA's range is finished there; a
//     unit cut by range boundaries leaves a normalised partial (o, lse) per
//     piece, merged by bd_decode_stream_combine_kernel.
//
// Roles: warps 0-3 softmax and epilogue (thread t = query row t = TMEM lane
// t), warp 4 TMA producer of Q and K, warp 5 MMA issuer, warp 6 TMA producer
// of V.  All roles enumerate the same segments in the same order; the K/V
// ring stage and the S/P/PV barrier phases follow one running tile counter
// across segments, so the Q load and S = QK^T of the next segment overlap
// the last PV and the epilogue of the current one.  TMEM holds kSBufs = 3
// S/P buffers (P, bf16, overwrites its own S) and one O; the forward issues
// QK two tiles ahead of PV, so the softmax warps find the next S ready.  Q
// is double-buffered in shared memory by segment parity (q_free: every QK of
// the segment that last used the buffer has retired); O is read out by the
// epilogue before the softmax of the next segment produces the P that its
// first PV needs (o_free).
#pragma once

#include "attn_tc.cuh"

namespace bd {

struct PParams {
    bf16 *out;
    float *lse;
    float *part_o;   // decode: [G][2][128][128] fp32 partial outputs
    float *part_lse; // decode: [G][2][128]
    int4 *cut_desc;  // decode: [G] unit cut at the end of CTA c's range:
                     // {rows (0: none), CTA of its last tile, out row, 0}
    const int32_t *cache_len;
    int B, Hq, Hkv, L, b;
    int d;         // head dim of q, k, v, out: 128, or 64 (read zero-extended to 128)
    int nkeys;     // key rows per kv-head: 2L or S_cap
    int mode;      // decode: 0 bidirectional, 1 causal
    int qtiles;    // fwd: 128-row query tiles per half
    int row_tiles; // decode: 128-row query tiles per unit
    int rows_unit; // decode: query rows per (sequence, kv-head) = group * b
    int sched_slot; // fwd: counter pair of this launch (0 .. kSchedSlots-1)
    int chunk;      // fwd: heads (head pairs in the paired kernel) per chunk of the work list
    float scale_log2;
};

struct Seg {
    int qhead, qrow0, nrows, kvhead;
    int lo0, hi0, lo1, hi1;     // key ranges
    int flo0, fhi0, flo1, fhi1; // keys every row of the tile sees
    int n0, nt;                 // tiles in range 0, in total
    int len;            // decode: cache length of the sequence
    int out_row0;       // decode: global output row of tile row 0
    int complete;       // decode: the segment covers its whole unit
    int slot;           // decode: partial slot (0 or 1) of this CTA
    int last_cta;       // decode: CTA holding the unit's last tile (cut
                        // units that start in this CTA's range), else -1
};
static_assert(sizeof(Seg) <= 128, "a decoded work item takes one 128-byte slot");

// Keys a decode row may see past the prefix: the block itself in modes 0
// and 1, nothing in mode 2 (cross-attention to the prefix only).
__device__ __forceinline__ int decode_own_keys(int b, int mode)
{
    return mode == 2 ? 0 : b;
}

// Number of 128-key tiles of one decode unit: -1 for an invalid length,
// 0 for an empty prefix in mode 2.
__device__ __forceinline__ int decode_unit_tiles(int len, int b, int S_cap, int mode)
{
    const int own = decode_own_keys(b, mode);
    if (len < 0 || (long long)len + own > S_cap)
        return -1;
    return (len + own + kTcN - 1) / kTcN;
}

// ----------------------------------------------------------------------------
// training / prefill work list

// The work items are handed out dynamically: the TMA producer of each CTA
// takes the next item index from a global counter and passes it to the MMA
// and softmax roles through a 4-entry ring in shared memory.  The heads are
// taken in chunks of p.chunk (the host sizes a chunk so that its K/V fit in
// half of L2); inside a chunk the list runs rank by rank (every head's
// heaviest query tile, then every head's next ...).  The CTAs running at any
// moment then share the K/V of the chunk in L2, and the list ends on the
// lightest tiles of its last chunk.  Head by head (one
// head's tiles heaviest first, then the next head's) the heaviest tiles of
// the last heads were handed out near the end: a list-scheduling model of
// the training shape puts the time lost to the tail at 7 % for the paired
// kernel, 3.5 % for the dQ pass, against under 2 % this way.  Each launch uses
// one of kSchedSlots counter pairs (rotating on the host); the last CTA of a
// launch to finish resets its pair.
constexpr int kSchedSlots = 64;

// Position w of a list of G groups x R ranks that runs chunk by chunk (C
// groups a chunk, the last one possibly smaller) and rank by rank inside a
// chunk: g = group, r = rank.
__device__ __forceinline__ void chunked_rank_order(int w, int G, int R, int C, int &g, int &r)
{
    const int c = w / (C * R);
    const int g0 = c * C;
    const int gc = min(C, G - g0);
    const int o = w - c * C * R;
    r = o / gc;
    g = g0 + o % gc;
}
// one-shot fault injection (see bd_attn_debug.h): CTA 0 skips one K copy
__device__ int g_fault_skip_k;
__device__ unsigned int g_sched_next[kSchedSlots];
__device__ unsigned int g_sched_done[kSchedSlots];
__device__ unsigned int g_sched_claim[kSchedSlots];

// Called once per CTA before its first fetch from counter pair `slot`.
// More claims than the launch has CTAs means that another launch uses the
// pair at the same time (the two then share the item counter and compute
// wrong results): that is recorded in the device status word.
__device__ __forceinline__ void sched_claim(int slot)
{
    if (atomicAdd(&g_sched_claim[slot], 1u) >= gridDim.x)
        raise_device_code(DEV_SCHED_OVERLAP);
}

// Called once per CTA after its last fetch: the launch's last CTA resets the
// pair for the next launch that draws it.
__device__ __forceinline__ void sched_finish(int slot)
{
    __threadfence();
    if (atomicAdd(&g_sched_done[slot], 1u) == gridDim.x - 1) {
        g_sched_next[slot] = 0;
        g_sched_done[slot] = 0;
        g_sched_claim[slot] = 0;
        __threadfence();
    }
}

struct FwdSource {
    __device__ void init(const PParams &) {}
    __device__ static long long items(const PParams &p)
    {
        return (long long)p.B * p.Hq * 2 * p.qtiles;
    }
    // item w: (batch, head) bh, cost rank r (0 = heaviest) in chunked rank order
    __device__ static void item(const PParams &p, int w, Seg &sg)
    {
        const int R = 2 * p.qtiles;
        int bh, r;
        chunked_rank_order(w, p.B * p.Hq, R, p.chunk, bh, r);
        const int idx = p.qtiles - 1 - (r >> 1);
        const int clean = r & 1; // noisy tile k is one K/V tile heavier
        sg.qrow0 = (clean ? p.L : 0) + idx * kTcM;
        sg.nrows = min(kTcM, p.L - idx * kTcM);
        sg.qhead = bh;
        sg.kvhead = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / (p.Hq / p.Hkv);
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
};

// ----------------------------------------------------------------------------
// block decode work list (stream-K over units x key tiles)

__device__ __forceinline__ long long range_start(long long T, int G, int c)
{
    return T * c / G;
}

// Whole-unit mode: when there are no more units than CTAs and the units are
// balanced (the longest at most 5/4 of the mean), CTA c streams unit c
// whole, so no unit is cut and nothing needs merging.  Otherwise the
// (unit, tile) space is cut into equal stream-K ranges.  Both kernels of a
// decode launch take this decision from the same device-resident lengths.
__device__ __forceinline__ bool decode_whole_units(const PParams &p, int G,
                                                   long long T, int maxt)
{
    const long long units = (long long)p.B * p.Hkv * p.row_tiles;
    return units <= G && (long long)maxt * units * 4 <= T * 5;
}

struct DecSource {
    bool whole;           // whole-unit mode (see decode_whole_units)
    long long t, t1, t0;  // position, end and start of this CTA's range
    long long T;          // tiles of the whole launch
    long long seq_base;   // first global tile of the current sequence
    int seq, seq_tiles, len;

    __device__ void load_seq(const PParams &p)
    {
        len = seq < p.B ? p.cache_len[seq] : 0;
        seq_tiles = seq < p.B ? max(0, decode_unit_tiles(len, p.b, p.nkeys, p.mode)) : 0;
    }
    __device__ void init(const PParams &p)
    {
        const int ups = p.Hkv * p.row_tiles; // units per sequence
        T = 0;
        int maxt = 0;
        for (int i = 0; i < p.B; ++i) {
            const int ti = max(0, decode_unit_tiles(p.cache_len[i], p.b, p.nkeys, p.mode));
            T += (long long)ups * ti;
            maxt = max(maxt, ti);
        }
        whole = decode_whole_units(p, gridDim.x, T, maxt);
        seq = 0;
        seq_base = 0;
        if (whole) {
            // CTA c takes unit c: its global tile range
            const int u = blockIdx.x;
            const int us = u / ups;
            long long base = 0;
            for (int i = 0; i < p.B && i < us; ++i)
                base += (long long)ups * max(0, decode_unit_tiles(p.cache_len[i], p.b, p.nkeys, p.mode));
            const int ti = us < p.B ? max(0, decode_unit_tiles(p.cache_len[us], p.b, p.nkeys, p.mode)) : 0;
            t0 = t = base + (long long)(u % ups) * ti;
            t1 = t + ti;
        } else {
            t0 = t = range_start(T, gridDim.x, blockIdx.x);
            t1 = range_start(T, gridDim.x, blockIdx.x + 1);
        }
        load_seq(p);
    }
    __device__ bool next(const PParams &p, Seg &sg)
    {
        if (t >= t1)
            return false;
        const int ups = p.Hkv * p.row_tiles;
        while (t >= seq_base + (long long)ups * seq_tiles) {
            seq_base += (long long)ups * seq_tiles;
            ++seq;
            load_seq(p);
        }
        const long long local = t - seq_base;
        const int uis = (int)(local / seq_tiles); // unit inside the sequence
        const int kt0 = (int)(local % seq_tiles);
        const long long left = t1 - t;
        const int n = (int)min((long long)(seq_tiles - kt0), left);
        const int g = uis / p.row_tiles, rt = uis % p.row_tiles;
        const int group = p.Hq / p.Hkv;
        sg.qhead = seq * p.Hkv + g;
        sg.kvhead = sg.qhead;
        sg.qrow0 = rt * kTcM;
        sg.nrows = min(kTcM, p.rows_unit - rt * kTcM);
        sg.lo0 = kt0 * kTcN;
        sg.hi0 = min((kt0 + n) * kTcN, len + decode_own_keys(p.b, p.mode));
        sg.lo1 = sg.hi1 = 0;
        sg.flo0 = 0;
        sg.fhi0 = len + (p.mode == 0 ? p.b : 0);
        sg.flo1 = sg.fhi1 = 0;
        sg.n0 = sg.nt = n;
        sg.len = len;
        sg.out_row0 = (seq * p.Hq + g * group) * p.b + rt * kTcM;
        sg.complete = (kt0 == 0 && n == seq_tiles);
        const long long u0 = seq_base + (long long)uis * seq_tiles;
        sg.slot = (u0 < t0) ? 0 : 1;
        // range x starts at floor(T x / G), so the last x starting at or
        // before tile e is floor(((e + 1) G - 1) / T)
        sg.last_cta = (!sg.complete && sg.slot == 1)
                          ? (int)(((u0 + seq_tiles) * gridDim.x - 1) / T)
                          : -1;
        t += n;
        return true;
    }
};

// ----------------------------------------------------------------------------

// KIND 0: training/prefill form, 1: block decode.  DH: head dim of the
// tensors, 128, or 64 / 32 read zero-extended to 128 columns (the QKs skip
// the zero K-steps; the columns of O past DH are computed but never written
// out).
template <int KIND, int DH>
__global__ void __launch_bounds__(kTcThreads, 1)
    bd_tc_persist_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const PParams p)
{
    typedef typename std::conditional<KIND == 0, FwdSource, DecSource>::type Src;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw_addr);

    const uint32_t bar0 = base + kSmemBar;
    const uint32_t bar_q = bar0; // Q buffer 0 landed
    auto bar_kfull = [&](int s) { return bar0 + 8 * (1 + s); };
    auto bar_vfull = [&](int s) { return bar0 + 8 * (1 + kTcStages + s); };
    // A K stage is free again once the QK that read it has completed, which
    // is what sfull of that tile tracks; a V stage once its PV has completed
    // (odone of that tile: two barriers for the two V stages).  So the
    // producers wait on those and the MMA thread commits nothing extra.
    static_assert(kTcStages == 2, "odone doubles as the V-stage release");
    const uint32_t bar_sfull0 = bar0 + 8 * (1 + 2 * kTcStages); // kSBufs
    const uint32_t bar_pfull0 = bar_sfull0 + 8 * kSBufs;        // kSBufs
    const uint32_t bar_odone0 = bar_pfull0 + 8 * kSBufs;        // 2
    const uint32_t bar_final = bar_odone0 + 16;
    const uint32_t bar_qfree0 = bar_final + 8;  // 2: Q buffer no longer read
    const uint32_t bar_ofree = bar_qfree0 + 16; // O read out by the epilogue
    const uint32_t bar_qfull1 = bar_ofree + 8;  // Q buffer 1 landed
    const uint32_t bar_ifull0 = bar_qfull1 + 8;   // 4: work item published
    const uint32_t bar_iempty0 = bar_ifull0 + 32; // 4: work item read by all roles
    static_assert(8 * (1 + 2 * kTcStages) + 16 * kSBufs + 16 + 8 + 16 + 8 + 8 + 64 <= 256,
                  "barriers overlap the item ring");
    volatile int *item_ring = reinterpret_cast<volatile int *>(sbase + kSmemBar + 256);
    Seg *seg_ring = reinterpret_cast<Seg *>(sbase + kSmemSeg);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + kSmemBar + 384);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sbase + kSmemBar + 392);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(bar_kfull(s), 1);
            mbar_init(bar_vfull(s), 1);
        }
        for (int i = 0; i < kSBufs; ++i) {
            mbar_init(bar_sfull0 + 8 * i, 1);
            mbar_init(bar_pfull0 + 8 * i, 128);
        }
        for (int i = 0; i < 2; ++i)
            mbar_init(bar_odone0 + 8 * i, 1);
        mbar_init(bar_final, 1);
        for (int i = 0; i < 2; ++i)
            mbar_init(bar_qfree0 + 8 * i, 1);
        mbar_init(bar_ofree, 128);
        mbar_init(bar_qfull1, 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar_ifull0 + 8 * i, 1);
            mbar_init(bar_iempty0 + 8 * i, 130); // MMA, V producer, 128 softmax threads
        }
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
    const uint32_t t_s0 = tmem;              // S/P buffers: columns [128 i, 128 i + 128)
    const uint32_t t_o = tmem + 128 * kSBufs; // O: columns [384, 512)
    auto bar_qfull = [&](int i) { return i ? bar_qfull1 : bar_q; };

    Src src;
    src.init(p);
    Seg sg;
    if constexpr (KIND == 1) {
        // the combine kernel may be scheduled now; it reads nothing of this
        // launch before the whole grid has finished
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        if (threadIdx.x == 0)
            p.cut_desc[blockIdx.x] = make_int4(0, 0, 0, 0);
        // an empty range (more CTAs than tiles) contributes an empty piece
        // to any cut unit that spans it
        if (src.t0 == src.t1 && threadIdx.x < kTcM)
            p.part_lse[(size_t)blockIdx.x * 2 * kTcM + threadIdx.x] = -INFINITY;
    }

    // Next segment of this CTA, identical for every role.  Training/prefill:
    // the producer takes the next item from the global counter, decodes it
    // (FwdSource::item: a few integer divisions) and publishes index and
    // decoded item in slot si % 4; the other roles copy it from there.
    // Decode: each role walks its static stream-K range.
    auto next_seg = [&](int si, bool producer, bool &ok) -> bool {
        if constexpr (KIND == 1) {
            return src.next(p, sg);
        } else {
        const int slot = si & 3;
        int w;
        if (producer) {
            if (si >= 4 && !(ok = mbar_wait(bar_iempty0 + 8 * slot,
                                             (uint32_t)(((si - 4) >> 2) & 1), abort_flag)))
                return false;
            if (si == 0)
                sched_claim(p.sched_slot);
            const unsigned int t = atomicAdd(&g_sched_next[p.sched_slot], 1u);
            w = (long long)t < FwdSource::items(p) ? (int)t : -1;
            if (w >= 0) {
                FwdSource::item(p, w, sg);
                seg_ring[slot] = sg;
            }
            item_ring[slot] = w;
            mbar_arrive(bar_ifull0 + 8 * slot);
        } else {
            if (!(ok = mbar_wait(bar_ifull0 + 8 * slot, (uint32_t)((si >> 2) & 1), abort_flag)))
                return false;
            w = item_ring[slot];
            if (w >= 0)
                sg = seg_ring[slot];
            mbar_arrive(bar_iempty0 + 8 * slot);
        }
        return w >= 0;
        }
    };

    if (warp == 4) {
        // ------------------------------------------- TMA producer: Q and K
        if (lane == 0) {
            bool ok = true;
            int si = 0;
            long long g = 0;   // running K/V tile counter
            long long kiss = 0;
            while (ok && next_seg(si, true, ok)) {
                // Q buffer si & 1 was last read by segment si - 2
                const int qbuf = si & 1;
                if (si >= 2 && !(ok = mbar_wait(bar_qfree0 + 8 * qbuf,
                                                 (uint32_t)(((si - 2) >> 1) & 1), abort_flag)))
                    break;
                mbar_expect_tx(bar_qfull(qbuf), kTileBytes);
                tma_load_3d(base + kSmemQ + qbuf * kTileBytes, &tm_q, 0, sg.qrow0,
                            sg.qhead, bar_qfull(qbuf));
                tma_load_3d(base + kSmemQ + qbuf * kTileBytes + kHalfTileBytes, &tm_q,
                            64, sg.qrow0, sg.qhead, bar_qfull(qbuf));
                ++si;
                for (int it = 0; it < sg.nt; ++it, ++g) {
                    const int ks = it < sg.n0 ? sg.lo0 + it * kTcN
                                              : sg.lo1 + (it - sg.n0) * kTcN;
                    const int s = (int)(g % kTcStages);
                    // stage s was last read by QK_{g-2}
                    if (g >= kTcStages) {
                        const long long gp = g - kTcStages;
                        if (!(ok = mbar_wait(bar_sfull0 + 8 * (int)(gp % kSBufs),
                                             (uint32_t)((gp / kSBufs) & 1), abort_flag)))
                            break;
                    }
                    if (g == 0 && blockIdx.x == 0 && atomicExch(&g_fault_skip_k, 0) != 0)
                        continue; // injected fault: this tile never arrives
                    mbar_expect_tx(bar_kfull(s), kTileBytes);
                    tma_load_3d(base + kSmemK + s * kTileBytes, &tm_k, 0, ks, sg.kvhead,
                                bar_kfull(s));
                    tma_load_3d(base + kSmemK + s * kTileBytes + kHalfTileBytes, &tm_k, 64,
                                ks, sg.kvhead, bar_kfull(s));
                    kiss = g + 1;
                }
            }
            if (KIND == 0) {
                // this CTA takes no more items; the last CTA resets the pair
                sched_finish(p.sched_slot);
            }
            // wait (bounded) for every copy this role issued
            const long long c0 = clock64();
            auto drain = [&](uint32_t bar, uint32_t par) {
                while (!mbar_try_wait(bar, par) && clock64() - c0 < kWaitCycles) {}
            };
            for (int x = si > 2 ? si - 2 : 0; x < si; ++x)
                drain(bar_qfull(x & 1), (uint32_t)((x >> 1) & 1));
            for (long long x = kiss > kTcStages ? kiss - kTcStages : 0; x < kiss; ++x)
                drain(bar_kfull((int)(x % kTcStages)), (uint32_t)((x / kTcStages) & 1));
        }
    } else if (warp == 6) {
        // ---------------------------------------------- TMA producer: V
        // A warp of its own, so a K load never queues behind a V load that
        // waits for its stage (and the other way round).
        if (lane == 0) {
            bool ok = true;
            int si = 0;
            long long g = 0;
            long long viss = 0;
            while (ok && next_seg(si, false, ok)) {
                ++si;
                for (int it = 0; it < sg.nt; ++it, ++g) {
                    const int ks = it < sg.n0 ? sg.lo0 + it * kTcN
                                              : sg.lo1 + (it - sg.n0) * kTcN;
                    const int s = (int)(g % kTcStages);
                    // stage s was last read by PV_{g-2}
                    if (g >= kTcStages &&
                        !(ok = mbar_wait(bar_odone0 + 8 * (int)(g & 1),
                                         (uint32_t)(((g - kTcStages) >> 1) & 1), abort_flag)))
                        break;
                    mbar_expect_tx(bar_vfull(s), kTileBytes);
                    tma_load_3d(base + kSmemV + s * kTileBytes, &tm_v, 0, ks, sg.kvhead,
                                bar_vfull(s));
                    tma_load_3d(base + kSmemV + s * kTileBytes + kHalfTileBytes, &tm_v, 64,
                                ks, sg.kvhead, bar_vfull(s));
                    viss = g + 1;
                }
            }
            const long long c0 = clock64();
            for (long long x = viss > kTcStages ? viss - kTcStages : 0; x < viss; ++x)
                while (!mbar_try_wait(bar_vfull((int)(x % kTcStages)),
                                      (uint32_t)((x / kTcStages) & 1)) &&
                       clock64() - c0 < kWaitCycles) {}
        }
    } else if (warp == 5) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(kTcM, kTcN, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(kTcM, kTcD, 1);
            bool ok = true;
            int si = 0;
            long long j = 0; // running tile counter
            auto issue_pv = [&](long long jg, bool first) -> bool {
                const int s = (int)(jg % kTcStages);
                const int b = (int)(jg % kSBufs);
                // O was last read out by the epilogue of segment si - 1
                if (first && si >= 1 &&
                    !mbar_wait(bar_ofree, (uint32_t)((si - 1) & 1), abort_flag))
                    return false;
                if (!mbar_wait(bar_pfull0 + 8 * b, (uint32_t)((jg / kSBufs) & 1), abort_flag))
                    return false;
                if (!mbar_wait(bar_vfull(s), (uint32_t)((jg / kTcStages) & 1), abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t vb = base + kSmemV + s * kTileBytes;
                const uint32_t tp = t_s0 + (uint32_t)b * 128;
#pragma unroll
                for (int kk = 0; kk < kTcN / 16; ++kk) {
                    uint64_t bdesc = smem_desc_sw128(vb + kk * 2048, kHalfTileBytes, 1024);
                    tc_mma_ts(t_o, tp + kk * 8, bdesc, idesc_pv, (!first || kk > 0) ? 1u : 0u);
                }
                tc_commit(bar_odone0 + 8 * (jg & 1));
                return true;
            };
            // Issue order QK_t, PV_{t-kLook} inside a segment; the last PVs
            // of a segment go out before the next segment's QKs, so its
            // epilogue is not held up by the next segment's loads.  Forward
            // (kLook = 2): with kSBufs = 3 S/P buffers the QK two tiles ahead
            // never waits for the softmax of tile t - 2, so the softmax warps
            // find the next S ready.  Decode (kLook = 1): HBM-bound, so PV
            // goes out as early as possible to turn the V ring over faster.
            // The buffer QK_t overwrites held P_{t-3}, whose PV was issued
            // before it (tcgen05.mma from one thread execute in issue order).
            constexpr int kLook = KIND == 0 ? 2 : 1;
            static_assert(kLook < kSBufs, "QK would overwrite a P not yet consumed");
            while (ok && next_seg(si, false, ok)) {
                if (!(ok = mbar_wait(bar_qfull(si & 1), (uint32_t)((si >> 1) & 1), abort_flag)))
                    break;
                tc_fence_after();
                for (int jj = 0; jj < sg.nt && ok; ++jj) {
                    const long long jg = j + jj;
                    const int s = (int)(jg % kTcStages);
                    if (!(ok = mbar_wait(bar_kfull(s), (uint32_t)((jg / kTcStages) & 1), abort_flag)))
                        break;
                    tc_fence_after();
                    const uint32_t kb = base + kSmemK + s * kTileBytes;
                    const uint32_t qb = base + kSmemQ + (si & 1) * kTileBytes;
                    const int b = (int)(jg % kSBufs);
                    const uint32_t ts = t_s0 + (uint32_t)b * 128;
#pragma unroll
                    for (int kk = 0; kk < kTcD / 16; ++kk) {
                        if (kk * 16 >= DH) // zero columns of a head dim below 128
                            break;
                        const uint32_t off = (kk >> 2) * kHalfTileBytes + (kk & 3) * 32;
                        tc_mma_ss(ts, smem_desc_sw128(qb + off, 16, 1024),
                                  smem_desc_sw128(kb + off, 16, 1024), idesc_qk,
                                  kk > 0 ? 1u : 0u);
                    }
                    tc_commit(bar_sfull0 + 8 * b);
                    if (jj == sg.nt - 1)
                        tc_commit(bar_qfree0 + 8 * (si & 1)); // Q buffer no longer read
                    if (jj >= kLook && !(ok = issue_pv(jg - kLook, jj == kLook)))
                        break;
                }
                for (int t = sg.nt > kLook ? sg.nt - kLook : 0; ok && t < sg.nt; ++t)
                    ok = issue_pv(j + t, t == 0);
                j += sg.nt;
                ++si;
            }
            tc_commit(bar_final);
            const long long c0 = clock64();
            while (!mbar_try_wait(bar_final, 0) && clock64() - c0 < kWaitCycles) {}
        }
    } else {
        // ---------------------------------------------------- softmax + epilogue
        const int row = threadIdx.x;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
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
            Span sp;
            if (KIND == 0) {
                sp = fwd_span(p.L, p.b, sg.qrow0 + rl);
            } else {
                const int jr = (sg.qrow0 + rl) % p.b;
                sp.a0 = 0;
                sp.a1 = sg.len + (p.mode == 0 ? p.b : p.mode == 1 ? jr + 1 : 0);
                sp.a2 = sp.a3 = 0;
            }
            float m_used = -INFINITY, l = 0.f;
            for (int jj = 0; jj < sg.nt; ++jj) {
                const long long jg = j + jj;
                const bool r0 = jj < sg.n0;
                const int ks = r0 ? sg.lo0 + jj * kTcN : sg.lo1 + (jj - sg.n0) * kTcN;
                const int khi = r0 ? sg.hi0 : sg.hi1;
                const int flo = r0 ? sg.flo0 : sg.flo1;
                const int fhi = r0 ? sg.fhi0 : sg.fhi1;
                const int sb = (int)(jg % kSBufs);
                ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull0 + 8 * sb,
                                                       (uint32_t)((jg / kSBufs) & 1), abort_flag));
                if (!ok)
                    break;
                tc_fence_after();
                const bool full = ks >= flo && ks + kTcN <= fhi && ks + kTcN <= khi;
                const long long jp = jg - 1; // PV_{jp} done => O stable
                // the FMA-pipe exponential relieves the special-function
                // unit where the softmax paces the tensor pipe (forward); the
                // HBM-bound decode measured faster without it
                ok = softmax_tile<KIND == 0 && kEmuExp2>(
                    t_s0 + (uint32_t)sb * 128 + lane_off, t_o + lane_off, full, sp, ks, khi, sl2,
                    jj >= 1, m_used, l, [&] {
                        return mbar_wait(bar_odone0 + 8 * (jp & 1), (uint32_t)((jp >> 1) & 1),
                                         abort_flag);
                    });
                if (!ok)
                    break;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_pfull0 + 8 * sb);
            }
            if (!ok)
                break;
            {
                // Wait for PV_{jl-1}, then PV_jl.  A parity wait is sound only
                // while its barrier is at most one phase short, and odone of
                // PV_jl last completed for PV_{jl-2}, which (issued after QK_jl
                // in the forward's order) may still run when this warp gets
                // here.  odone of PV_{jl-1} last completed for PV_{jl-3},
                // issued before QK_jl and so finished; once PV_{jl-1} is done,
                // so is PV_{jl-2}.
                const long long jl = j + sg.nt - 1; // last PV of the segment
                ok = jl < 1 || __all_sync(0xffffffffu,
                                          mbar_wait(bar_odone0 + 8 * ((jl - 1) & 1),
                                                    (uint32_t)(((jl - 1) >> 1) & 1), abort_flag));
                ok = ok && __all_sync(0xffffffffu,
                                      mbar_wait(bar_odone0 + 8 * (jl & 1),
                                                (uint32_t)((jl >> 1) & 1), abort_flag));
                if (!ok)
                    break;
                tc_fence_after();
            }
            // ------------------------------------------------ epilogue
            const bool valid = row < sg.nrows;
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            const float lse_v = (l > 0.f) ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
            const bool to_out = (KIND == 0) || sg.complete;
            size_t grow;
            if (KIND == 0)
                grow = (size_t)sg.qhead * 2 * p.L + sg.qrow0 + row;
            else
                grow = (size_t)sg.out_row0 + row;
            const size_t prow = ((size_t)blockIdx.x * 2 + sg.slot) * kTcM + row;
            // Forward: output rows go through this warp's staging area so
            // that each global store writes two whole rows (512 contiguous
            // bytes) instead of one 16-byte piece of 32 rows.  Chunk c (16
            // bytes) of row l sits at l * 256 + ((c ^ (l & 7)) << 4):
            // conflict-free both for a lane writing its own row and for 16
            // lanes reading one row.  (Decode writes few output tiles per
            // CTA; it keeps the per-row stores.)
            constexpr bool kStage = KIND == 0;
            const uint32_t epi = base + kSmemEpi + (uint32_t)warp * (32 * 256);
#pragma unroll
            for (int q4 = 0; q4 < kTcD / 32; ++q4) {
                if (q4 * 32 >= DH) // O columns past the head dim are not output
                    break;
                uint32_t o[32];
                tmem_ld32_wait(t_o + lane_off + q4 * 32, o);
                if (kStage) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        const uint32_t c = (uint32_t)(q4 * 4 + i / 8);
                        const uint32_t a = epi + (uint32_t)lane * 256 + ((c ^ (uint32_t)(lane & 7)) << 4);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                                     "r"(pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv)),
                                     "r"(pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv)),
                                     "r"(pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv)),
                                     "r"(pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv))
                                     : "memory");
                    }
                } else if (valid && to_out) {
                    uint4 *orow = reinterpret_cast<uint4 *>(p.out + grow * DH);
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v4;
                        v4.x = pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
                        v4.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                        v4.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                        v4.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                        orow[q4 * 4 + i / 8] = v4;
                    }
                } else if (valid) {
                    float4 *prow4 = reinterpret_cast<float4 *>(p.part_o + prow * kTcD);
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        prow4[q4 * 8 + i / 4] = make_float4(
                            __uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                            __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                }
            }
            if (kStage) {
                __syncwarp();
                const size_t row0 = grow - (size_t)row + (size_t)warp * 32; // this warp's first row
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const int r = 2 * i + (lane >> 4); // row within the warp's 32
                    const uint32_t cc = (uint32_t)(lane & 15);
                    uint32_t x0, x1, x2, x3;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
                                 : "r"(epi + (uint32_t)r * 256 + ((cc ^ (uint32_t)(r & 7)) << 4))
                                 : "memory");
                    if (warp * 32 + r < sg.nrows && (int)cc * 8 < DH)
                        reinterpret_cast<uint4 *>(p.out + (row0 + r) * DH)[cc] =
                            make_uint4(x0, x1, x2, x3);
                }
                __syncwarp();
            }
            if (valid) {
                if (to_out)
                    p.lse[grow] = lse_v;
                else
                    p.part_lse[prow] = lse_v;
            }
            if (KIND == 1 && !to_out && sg.last_cta >= 0 && row == 0)
                p.cut_desc[blockIdx.x] = make_int4(sg.nrows, sg.last_cta, sg.out_row0, 0);
            tc_fence_before();
            mbar_arrive(bar_ofree);
            j += sg.nt;
            ++si;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

// Merges the partial results of decode units cut by stream-K range
// boundaries, and writes NaN rows for sequences with an invalid cache
// length.  The attention kernel leaves, for every CTA c whose range ends
// inside a unit that started in it, a descriptor: the unit's rows, its output
// row and the CTA x_e holding its last tile.  The unit's pieces are slot 1 of
// CTA c and slot 0 of CTAs c + 1 .. x_e (an empty range holds an empty
// piece).  Grid (G, kCombineRowGroups): CTA (c, rg) merges rows
// rg * 32 .. rg * 32 + 31 of the unit of descriptor c, warp w taking four
// rows and lane l output columns 4l .. 4l + 3, so every load is coalesced and
// the four rows' loads are independent.  Launched as a programmatic
// dependent of the attention kernel: it may start while that kernel runs,
// and waits for it to finish before reading anything it wrote.
constexpr int kCombineRowsPerWarp = 4;
constexpr int kCombineRowGroups = kTcM / (8 * kCombineRowsPerWarp);

__global__ void __launch_bounds__(256)
    bd_decode_stream_combine_kernel(const PParams p)
{
    const int c = blockIdx.x, rg = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int R = kCombineRowsPerWarp;

    if (rg == 0) { // sequences with no key tile (i % G == c), for which the
                   // attention kernel writes nothing: an invalid length gives
                   // NaN rows, an empty prefix in mode 2 rows with no visible
                   // key (out 0, lse -inf)
        for (int i = c; i < p.B; i += gridDim.x) {
            const int tiles = decode_unit_tiles(p.cache_len[i], p.b, p.nkeys, p.mode);
            if (tiles > 0)
                continue;
            const float fill = tiles < 0 ? NAN : 0.f;
            const float lfill = tiles < 0 ? NAN : -INFINITY;
            for (int r = threadIdx.x; r < p.Hq * p.b; r += blockDim.x) {
                const size_t orow = (size_t)i * p.Hq * p.b + r;
                for (int t = 0; t < p.d; ++t)
                    p.out[orow * p.d + t] = __float2bfloat16_rn(fill);
                p.lse[orow] = lfill;
            }
            if (threadIdx.x == 0 && tiles < 0)
                raise_device_code(DEV_BAD_CACHE_LEN);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int4 desc = p.cut_desc[c];
    const int nrows = desc.x, last = desc.y;
    const int r0 = (rg * 8 + warp) * R;
    if (r0 >= nrows)
        return;
    float m[R], z[R];
    float4 acc[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        m[k] = -INFINITY;
        z[k] = 0.f;
        acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int x = c; x <= last; ++x) {
        const size_t pr0 = ((size_t)x * 2 + (x == c ? 1 : 0)) * kTcM + r0;
        float ls[R];
        float4 v[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            ls[k] = p.part_lse[pr0 + k];
            v[k] = reinterpret_cast<const float4 *>(p.part_o + (pr0 + k) * kTcD)[lane];
        }
#pragma unroll
        for (int k = 0; k < R; ++k) {
            if (r0 + k >= nrows || ls[k] == -INFINITY)
                continue; // no row here, or no visible key in this piece
            const float mn = fmaxf(m[k], ls[k]);
            const float a = ex2((m[k] - mn) * kLog2e); // 0 while m is -inf
            const float w = ex2((ls[k] - mn) * kLog2e);
            z[k] = z[k] * a + w;
            acc[k].x = acc[k].x * a + w * v[k].x;
            acc[k].y = acc[k].y * a + w * v[k].y;
            acc[k].z = acc[k].z * a + w * v[k].z;
            acc[k].w = acc[k].w * a + w * v[k].w;
            m[k] = mn;
        }
    }
#pragma unroll
    for (int k = 0; k < R; ++k) {
        if (r0 + k >= nrows)
            break;
        const size_t orow = (size_t)desc.z + r0 + k;
        const float inv = z[k] > 0.f ? 1.f / z[k] : 0.f;
        uint2 o2;
        o2.x = pack_bf16x2(acc[k].x * inv, acc[k].y * inv);
        o2.y = pack_bf16x2(acc[k].z * inv, acc[k].w * inv);
        if (lane * 4 < p.d)
            reinterpret_cast<uint2 *>(p.out + orow * p.d)[lane] = o2;
        if (lane == 0)
            p.lse[orow] = z[k] > 0.f ? m[k] + __logf(z[k]) : -INFINITY;
    }
}

} // namespace bd
