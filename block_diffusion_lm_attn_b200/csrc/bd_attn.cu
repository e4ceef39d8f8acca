// C-ABI entry points of libbdattn.so: argument validation, launch planning
// and kernel launches on the caller's stream.  See include/bd_attn.h for the
// contract of each call.
//
// Kernels, all tcgen05 (head dims 64 and 32 on tiles zero-extended to 128
// columns): the forward on the paired kernel (attn_tc_pair.cuh) when the GQA
// group is even, else on the one-tile persistent kernel (attn_tc_persist.cuh),
// which also runs block decode; the backward in attn_tc_bwd.cuh; the cache
// and SPRINT kernels in cache_ops.cuh.
#include "bd_attn.h"
#include "bd_attn_debug.h"

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <algorithm>
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "attn_tc.cuh"
#include "attn_tc_persist.cuh"
#include "attn_tc_pair.cuh"
#include "attn_tc_bwd.cuh"
#include "bd_common.cuh"
#include "cache_ops.cuh"

namespace {

using bd::bf16;

// B200 SM count: the persistent grids and the decode workspace are sized
// for at most this many CTAs.
constexpr int kMaxGrid = 148;

inline bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

inline bool supported_d(int d) { return d == 32 || d == 64 || d == 128; }

inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// The paired forward kernel moves registers between its warpgroups with
// setmaxnreg, which can only hand out what the CTA was launched with: use it
// only if the compiled kernel's per-thread registers cover the split (a
// warpgroup asking for more than exists would wait for ever).
template <int DH>
bool pair_kernel_usable()
{
    static std::atomic<int> usable{-1};
    int u = usable.load();
    if (u < 0) {
        cudaFuncAttributes a;
        cudaFuncAttributes b;
        const long long need = 2LL * 128 * bd::kPairRegsSoftmax + 128LL * bd::kPairRegsOther;
        u = (cudaFuncGetAttributes(&a, bd::bd_tc_pair_kernel<DH, true>) == cudaSuccess &&
             cudaFuncGetAttributes(&b, bd::bd_tc_pair_kernel<DH, false>) == cudaSuccess &&
             (long long)a.numRegs * bd::kPairThreads >= need &&
             (long long)b.numRegs * bd::kPairThreads >= need)
                ? 1
                : 0;
        usable.store(u);
    }
    return u == 1;
}

bool pair_kernel_usable(int d)
{
    return d == 64 ? pair_kernel_usable<64>()
                   : d == 32 ? pair_kernel_usable<32>() : pair_kernel_usable<128>();
}

// Grid cap set by bd_attn_debug_set_grid (0: none).
std::atomic<int> g_grid_cap{0};

int persistent_grid()
{
    int dev = 0, sms = kMaxGrid;
    int g = kMaxGrid;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) ==
            cudaSuccess &&
        sms > 0)
        g = sms < kMaxGrid ? sms : kMaxGrid;
    const int cap = g_grid_cap.load();
    return cap > 0 && cap < g ? cap : g;
}

// Groups (heads, or head pairs) per chunk of a forward or dQ work list: as
// many as keep the bytes the chunk's CTAs share in L2 (the K/V a group
// reads) within half of B200's 126 MB L2, and at least one.  A chunk runs
// heaviest rank first, so the larger it is, the lighter the items that end
// the list (a list-scheduling model of the training shape: 98.2 % of the
// balanced time with 16 head pairs a chunk, 99.5 % with 32 or more).
// Chunk size set by bd_attn_debug_set_chunk (0: the defaults).
std::atomic<int> g_chunk_fixed{0};

int list_chunk(long long bytes_per_group, long long groups)
{
    const int fixed = g_chunk_fixed.load();
    if (fixed > 0)
        return (int)std::max(1LL, std::min((long long)fixed, groups));
    constexpr long long kBudget = 64LL << 20;
    const long long c = bytes_per_group > 0 ? kBudget / bytes_per_group : groups;
    return (int)std::max(1LL, std::min(c, groups));
}

// Decode launch plan.  A pure function of the sizes, so the workspace query
// and the launch agree without a device round trip: stream-K over (unit, key
// tile) on <= kMaxGrid persistent CTAs (d = 64 and 32 on tiles zero-extended
// to 128 columns); scratch = 2 partial (o, lse) slots of 128 rows x 128
// columns per CTA and a cut descriptor per CTA, whatever the sizes.
struct DecodePlan {
    int row_tiles;
    size_t rows_all, o_bytes, lse_bytes, desc_bytes, total_bytes;
};

bool decode_plan(int B, int Hq, int Hkv, int b, int d, int S_cap,
                 DecodePlan &pl)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || b <= 0 || d <= 0 || S_cap <= 0 ||
        Hq % Hkv != 0)
        return false;
    const long long rows = (long long)(Hq / Hkv) * b;
    pl.rows_all = (size_t)B * Hq * b;
    pl.row_tiles = (int)cdiv(rows, bd::kTcM);
    pl.o_bytes = round256((size_t)kMaxGrid * 2 * bd::kTcM * bd::kTcD * sizeof(float));
    pl.lse_bytes = round256((size_t)kMaxGrid * 2 * bd::kTcM * sizeof(float));
    pl.desc_bytes = round256((size_t)kMaxGrid * sizeof(int4));
    pl.total_bytes = pl.o_bytes + pl.lse_bytes + pl.desc_bytes;
    return true;
}

// Per-device internal decode workspace (workspace == NULL).  A buffer once
// handed out is never freed: a CUDA graph captured earlier may still hold
// its address.  When a call needs more, a larger buffer is allocated and
// becomes the current one; the smaller ones stay allocated (and valid for
// the graphs that recorded them) until the process exits.
struct InternalWorkspace {
    std::mutex mu;
    void *ptr[64] = {};
    size_t bytes[64] = {};
};
InternalWorkspace g_ws;

bd_status get_internal_workspace(size_t need, void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return BD_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_ws.mu);
    if (g_ws.bytes[dev] < need) {
        void *p = nullptr;
        if (cudaMalloc(&p, need) != cudaSuccess)
            return BD_ERR_CUDA;
        g_ws.ptr[dev] = p; // the previous buffer is kept, not freed
        g_ws.bytes[dev] = need;
    }
    *out = g_ws.ptr[dev];
    return BD_OK;
}

// Raises the kernel's dynamic shared-memory limit once per device (the
// attribute is per device; later calls, including ones made while a stream
// is being captured, skip the runtime call).
template <auto Kernel> bd_status set_smem(int bytes)
{
    static std::atomic<unsigned long long> done{0}; // one per kernel
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return BD_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit)
        return BD_OK;
    if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess)
        return BD_ERR_CUDA;
    done.fetch_or(bit, std::memory_order_acq_rel);
    return BD_OK;
}

// cuTensorMapEncodeTiled, fetched once through the runtime's driver entry
// point (no link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p,
                                    cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D map over a row-major bf16 tensor [n2][n1][128]: boxes of 64 columns x
// box_rows rows x 1, 128-byte swizzle, rows beyond n1 read as zero.
bool make_map_rows(CUtensorMap *m, const void *base, uint64_t n1, uint64_t n2,
                   uint32_t box_rows, uint64_t d = 128)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return false;
    // rows of d bf16 (d = 64 or 128) read as 64-column boxes; with d = 64 the
    // box at column 64 lies wholly outside the tensor and reads as zeros, so
    // the head-dim-128 kernels run unchanged on a zero-extended tile
    cuuint64_t dims[3] = {d, n1, n2};
    cuuint64_t strides[2] = {d * 2, d * 2 * n1};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                     const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_map_rows128(CUtensorMap *m, const void *base, uint64_t n1,
                      uint64_t n2, uint64_t d = 128)
{
    return make_map_rows(m, base, n1, n2, 128, d);
}

// Counter pair of the next persistent launch that hands out work items
// dynamically (forward, and both backward passes).
std::atomic<unsigned int> g_launches{0};
int next_sched_slot()
{
    return (int)(g_launches.fetch_add(1u) % bd::kSchedSlots);
}

template <int KIND, int DH>
bd_status launch_persist_dh(const CUtensorMap &mq, const CUtensorMap &mk,
                            const CUtensorMap &mv, const bd::PParams &p, int grid,
                            cudaStream_t st)
{
    auto kern = bd::bd_tc_persist_kernel<KIND, DH>;
    if (set_smem<bd::bd_tc_persist_kernel<KIND, DH>>(bd::kTcSmemBytes) != BD_OK)
        return BD_ERR_CUDA;
    kern<<<grid, bd::kTcThreads, bd::kTcSmemBytes, st>>>(mq, mk, mv, p);
    return cudaGetLastError() == cudaSuccess ? BD_OK : BD_ERR_CUDA;
}

template <int DH, bool EMU>
bd_status launch_pair_emu(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                          const bd::PParams &p, int grid, cudaStream_t st)
{
    if (set_smem<bd::bd_tc_pair_kernel<DH, EMU>>(bd::kPairSmemBytes) != BD_OK)
        return BD_ERR_CUDA;
    bd::bd_tc_pair_kernel<DH, EMU><<<grid, bd::kPairThreads, bd::kPairSmemBytes, st>>>(mq, mk,
                                                                                       mv, p);
    return cudaGetLastError() == cudaSuccess ? BD_OK : BD_ERR_CUDA;
}

template <int DH>
bd_status launch_pair(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                      const bd::PParams &p, int grid, cudaStream_t st)
{
    return p.qtiles >= bd::kPairEmuQtiles ? launch_pair_emu<DH, true>(mq, mk, mv, p, grid, st)
                                          : launch_pair_emu<DH, false>(mq, mk, mv, p, grid, st);
}

template <int KIND>
bd_status launch_persist(const CUtensorMap &mq, const CUtensorMap &mk,
                         const CUtensorMap &mv, const bd::PParams &p, int grid,
                         cudaStream_t st)
{
    return p.d == 64   ? launch_persist_dh<KIND, 64>(mq, mk, mv, p, grid, st)
           : p.d == 32 ? launch_persist_dh<KIND, 32>(mq, mk, mv, p, grid, st)
                       : launch_persist_dh<KIND, 128>(mq, mk, mv, p, grid, st);
}

// Host-side checks shared by both decode entry points.
bd_status decode_validate(const void *q_blk, const void *k_cache,
                          const void *v_cache, const int32_t *cache_len,
                          const void *out, const float *lse, int B, int Hq,
                          int Hkv, int b, int d, int mode, int S_cap,
                          DecodePlan &pl)
{
    if (!q_blk || !k_cache || !v_cache || !cache_len || !out || !lse)
        return BD_ERR_INVALID_ARG;
    if (!aligned16(q_blk) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(out) || !aligned16(lse) ||
        (reinterpret_cast<uintptr_t>(cache_len) & 3u))
        return BD_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || b <= 0 || d <= 0 || S_cap <= 0)
        return BD_ERR_INVALID_ARG;
    if (mode < 0 || mode > 2)
        return BD_ERR_INVALID_ARG;
    // modes 0 and 1 read the block's own keys after the prefix
    if (Hq % Hkv != 0 || (mode != 2 && S_cap < b))
        return BD_ERR_INVALID_ARG;
    if (!supported_d(d))
        return BD_ERR_UNSUPPORTED;
    if (!decode_plan(B, Hq, Hkv, b, d, S_cap, pl))
        return BD_ERR_INVALID_ARG;
    if ((long long)B * Hkv > 65535LL || pl.row_tiles > 65535 ||
        (long long)B * Hkv * pl.row_tiles > (1LL << 30))
        return BD_ERR_UNSUPPORTED;
    return BD_OK;
}

// Launches block decode with a validated plan and a workspace of at least
// pl.total_bytes (256-byte aligned).
bd_status decode_launch(const void *q_blk, const void *k_cache,
                        const void *v_cache, const int32_t *cache_len,
                        void *out, float *lse, int B, int Hq, int Hkv, int b,
                        int d, int mode, cudaStream_t stream, int S_cap,
                        void *workspace, const DecodePlan &pl)
{
    float *part_o = static_cast<float *>(workspace);
    float *part_lse =
        reinterpret_cast<float *>(static_cast<char *>(workspace) + pl.o_bytes);
    const float scale_log2 = (1.0f / std::sqrt((float)d)) * bd::kLog2e;
    {
        bd::PParams p = {};
        p.out = static_cast<bf16 *>(out);
        p.lse = lse;
        p.part_o = part_o;
        p.part_lse = part_lse;
        p.cut_desc = reinterpret_cast<int4 *>(static_cast<char *>(workspace) + pl.o_bytes +
                                              pl.lse_bytes);
        p.cache_len = cache_len;
        p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = 0; p.b = b;
        p.d = d;
        p.nkeys = S_cap;
        p.mode = mode;
        p.row_tiles = pl.row_tiles;
        p.rows_unit = (Hq / Hkv) * b;
        p.scale_log2 = scale_log2;
        CUtensorMap mq, mk, mv;
        if (!make_map_rows128(&mq, q_blk, (uint64_t)p.rows_unit, (uint64_t)B * Hkv, d) ||
            !make_map_rows128(&mk, k_cache, (uint64_t)S_cap, (uint64_t)B * Hkv, d) ||
            !make_map_rows128(&mv, v_cache, (uint64_t)S_cap, (uint64_t)B * Hkv, d))
            return BD_ERR_CUDA;
        const int G = persistent_grid();
        bd_status st = launch_persist<1>(mq, mk, mv, p, G, stream);
        if (st != BD_OK)
            return st;
        // programmatic dependent launch: the combine's blocks may be placed
        // while the attention kernel runs; they wait for its end in-kernel
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(G, bd::kCombineRowGroups);
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, bd::bd_decode_stream_combine_kernel, p) != cudaSuccess)
            return BD_ERR_CUDA;
        return cudaGetLastError() == cudaSuccess ? BD_OK : BD_ERR_CUDA;
    }
}

} // namespace

extern "C" {

const char *bd_attn_status_string(bd_status s)
{
    switch (s) {
    case BD_OK: return "ok";
    case BD_ERR_INVALID_ARG: return "invalid argument";
    case BD_ERR_UNSUPPORTED: return "unsupported configuration";
    case BD_ERR_CUDA: return "CUDA error";
    case BD_ERR_DEVICE_TIMEOUT:
        return "device-side check failed (bounded wait ran out or bad size)";
    }
    return "unknown status";
}

bd_status bd_attn_fwd(const void *q, const void *k, const void *v, void *out,
                      float *lse, int B, int Hq, int Hkv, int L, int b, int d,
                      float scale, cudaStream_t stream)
{
    if (!q || !k || !v || !out || !lse)
        return BD_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        !aligned16(lse))
        return BD_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || b <= 0 || d <= 0)
        return BD_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || L % b != 0)
        return BD_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale))
        return BD_ERR_INVALID_ARG;
    if (!supported_d(d))
        return BD_ERR_UNSUPPORTED;
    if ((long long)B * Hq > 65535LL || 2LL * L * (long long)B * Hq * d > (1LL << 40))
        return BD_ERR_UNSUPPORTED;

    {
        // tcgen05 kernels; d = 64 and 32 run on tiles zero-extended to 128
        // columns
        bd::PParams p = {};
        p.out = static_cast<bf16 *>(out);
        p.lse = lse;
        p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.b = b;
        p.d = d;
        p.nkeys = 2 * L;
        p.qtiles = (int)cdiv(L, bd::kTcM);
        p.scale_log2 = scale * bd::kLog2e;
        // heads of one kv-head share its K/V: 2 x 2L x d bf16
        const long long kv_bytes = 8LL * L * d;
        CUtensorMap mq, mk, mv;
        const uint64_t N = 2ull * L;
        if (!make_map_rows128(&mq, q, N, (uint64_t)B * Hq, d) ||
            !make_map_rows128(&mk, k, N, (uint64_t)B * Hkv, d) ||
            !make_map_rows128(&mv, v, N, (uint64_t)B * Hkv, d))
            return BD_ERR_CUDA;
        p.sched_slot = next_sched_slot();
        // two query heads of one GQA group per CTA when the group size is even
        const bool pair = (Hq / Hkv) % 2 == 0 && pair_kernel_usable(d);
        const long long items = (long long)B * (pair ? Hq / 2 : Hq) * 2 * p.qtiles;
        p.chunk = pair ? list_chunk(kv_bytes / ((Hq / Hkv) / 2), (long long)B * (Hq / 2))
                       : list_chunk(kv_bytes / (Hq / Hkv), (long long)B * Hq);
        int G = persistent_grid();
        if (items < G)
            G = (int)items;
        if (pair)
            return d == 64   ? launch_pair<64>(mq, mk, mv, p, G, stream)
                   : d == 32 ? launch_pair<32>(mq, mk, mv, p, G, stream)
                             : launch_pair<128>(mq, mk, mv, p, G, stream);
        return launch_persist<0>(mq, mk, mv, p, G, stream);
    }
}

size_t bd_attn_bwd_workspace_bytes(int B, int Hq, int L)
{
    if (B <= 0 || Hq <= 0 || L <= 0)
        return 0;
    return 2 * round256((size_t)B * Hq * 2 * L * sizeof(float));
}

bd_status bd_attn_bwd(const void *q, const void *k, const void *v,
                      const void *out, const float *lse, const void *dout,
                      void *dq, void *dk, void *dv, int B, int Hq, int Hkv,
                      int L, int b, int d, float scale, cudaStream_t stream,
                      void *workspace, size_t workspace_bytes)
{
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace)
        return BD_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        !aligned16(lse) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return BD_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || b <= 0 || d <= 0)
        return BD_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || L % b != 0)
        return BD_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale))
        return BD_ERR_INVALID_ARG;
    if (workspace_bytes < bd_attn_bwd_workspace_bytes(B, Hq, L))
        return BD_ERR_INVALID_ARG;
    if (d != 128)
        return BD_ERR_UNSUPPORTED;
    if ((long long)B * Hq > 65535LL || 2LL * L * (long long)B * Hq * d > (1LL << 40))
        return BD_ERR_UNSUPPORTED;

    bd::BParams p = {};
    p.out = static_cast<const bf16 *>(out);
    p.dout = static_cast<const bf16 *>(dout);
    p.lse = lse;
    const size_t rows = (size_t)B * Hq * 2 * L;
    p.D = static_cast<float *>(workspace);
    p.lse2 = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                       round256(rows * sizeof(float)));
    p.dq = static_cast<bf16 *>(dq);
    p.dk = static_cast<bf16 *>(dk);
    p.dv = static_cast<bf16 *>(dv);
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.b = b;
    p.qtiles = (int)cdiv(L, bd::kTcM);
    p.chunk_q = list_chunk(8LL * L * d / (Hq / Hkv), (long long)B * Hq);
    const int fixed = g_chunk_fixed.load();
    p.chunk_kv = fixed > 0 ? fixed : bd::kBwdChunkGroups;
    p.scale = scale;
    p.scale_log2 = scale * bd::kLog2e;

    CUtensorMap mq, mq_step, mdo, mdo_step, mk, mv;
    const uint64_t N = 2ull * L;
    if (!make_map_rows(&mq, q, N, (uint64_t)B * Hq, 128) ||
        !make_map_rows(&mq_step, q, N, (uint64_t)B * Hq, bd::kBwdSub) ||
        !make_map_rows(&mdo, dout, N, (uint64_t)B * Hq, 128) ||
        !make_map_rows(&mdo_step, dout, N, (uint64_t)B * Hq, bd::kBwdSub) ||
        !make_map_rows(&mk, k, N, (uint64_t)B * Hkv, 128) ||
        !make_map_rows(&mv, v, N, (uint64_t)B * Hkv, 128))
        return BD_ERR_CUDA;

    bd::bd_bwd_prep_kernel<<<(unsigned)((rows + bd::kPrepRowsPerBlock - 1) / bd::kPrepRowsPerBlock),
                             256, 0, stream>>>(p, (long long)rows);
    if (cudaGetLastError() != cudaSuccess)
        return BD_ERR_CUDA;

    const int G0 = persistent_grid();
    {
        p.sched_slot = next_sched_slot();
        const long long items = (long long)B * Hkv * 2 * p.qtiles;
        const int G = items < G0 ? (int)items : G0;
        if (set_smem<bd::bd_bwd_dkdv_kernel>(bd::kKvSmemBytes) != BD_OK)
            return BD_ERR_CUDA;
        bd::bd_bwd_dkdv_kernel<<<G, bd::kBwdThreads, bd::kKvSmemBytes, stream>>>(mk, mv, mq_step,
                                                                               mdo_step, p);
        if (cudaGetLastError() != cudaSuccess)
            return BD_ERR_CUDA;
    }
    {
        p.sched_slot = next_sched_slot();
        const long long items = (long long)B * Hq * 2 * p.qtiles;
        const int G = items < G0 ? (int)items : G0;
        if (set_smem<bd::bd_bwd_dq_kernel>(bd::kDqSmemBytes) != BD_OK)
            return BD_ERR_CUDA;
        bd::bd_bwd_dq_kernel<<<G, bd::kBwdThreads, bd::kDqSmemBytes, stream>>>(mq, mdo, mk, mv,
                                                                             p);
    }
    return cudaGetLastError() == cudaSuccess ? BD_OK : BD_ERR_CUDA;
}

size_t bd_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int b, int d,
                                      int S_cap)
{
    DecodePlan pl;
    if (!decode_plan(B, Hq, Hkv, b, d, S_cap, pl))
        return 0;
    return pl.total_bytes;
}

bd_status bd_attn_decode(const void *q_blk, const void *k_cache,
                         const void *v_cache, const int32_t *cache_len,
                         void *out, float *lse, int B, int Hq, int Hkv, int b,
                         int d, int intra_block_mode, cudaStream_t stream,
                         int S_cap, void *workspace, size_t workspace_bytes)
{
    DecodePlan pl;
    bd_status st = decode_validate(q_blk, k_cache, v_cache, cache_len, out,
                                   lse, B, Hq, Hkv, b, d, intra_block_mode,
                                   S_cap, pl);
    if (st != BD_OK)
        return st;
    if (workspace) {
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) ||
            workspace_bytes < pl.total_bytes)
            return BD_ERR_INVALID_ARG;
    } else {
        st = get_internal_workspace(pl.total_bytes, &workspace);
        if (st != BD_OK)
            return st;
    }
    return decode_launch(q_blk, k_cache, v_cache, cache_len, out, lse, B, Hq,
                         Hkv, b, d, intra_block_mode, stream, S_cap, workspace,
                         pl);
}

bd_status bd_spec_accept(const int32_t *draft, const int32_t *target,
                         int32_t *n_accept, int B, int b, cudaStream_t stream)
{
    if (!draft || !target || !n_accept || B <= 0 || b <= 0)
        return BD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(draft) | reinterpret_cast<uintptr_t>(target) |
         reinterpret_cast<uintptr_t>(n_accept)) & 3u)
        return BD_ERR_INVALID_ARG;
    bd::bd_spec_accept_kernel<<<(B + 7) / 8, 256, 0, stream>>>(draft, target,
                                                               n_accept, B, b);
    return cudaGetLastError() == cudaSuccess ? BD_OK : BD_ERR_CUDA;
}

bd_status bd_cache_append(void *k_cache, void *v_cache, int32_t *cache_len,
                          const void *k_new, const void *v_new,
                          const int32_t *n_new, int B, int Hkv, int b, int d,
                          int S_cap, cudaStream_t stream)
{
    if (!k_cache || !v_cache || !cache_len || !n_new || (!k_new != !v_new))
        return BD_ERR_INVALID_ARG;
    if (B <= 0 || Hkv <= 0 || b <= 0 || d <= 0 || S_cap <= 0)
        return BD_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) || (k_new && !aligned16(k_new)) ||
        (v_new && !aligned16(v_new)) ||
        ((reinterpret_cast<uintptr_t>(cache_len) | reinterpret_cast<uintptr_t>(n_new)) & 3u))
        return BD_ERR_INVALID_ARG;
    if (!supported_d(d))
        return BD_ERR_UNSUPPORTED;
    bd::bd_cache_append_kernel<<<B, 512, 0, stream>>>(
        static_cast<bf16 *>(k_cache), static_cast<bf16 *>(v_cache), cache_len,
        static_cast<const bf16 *>(k_new), static_cast<const bf16 *>(v_new), n_new, Hkv, b,
        d, S_cap);
    return cudaGetLastError() == cudaSuccess ? BD_OK : BD_ERR_CUDA;
}

bd_status bd_cache_crop(int32_t *cache_len, int B, int max_len,
                        cudaStream_t stream)
{
    if (!cache_len || B <= 0 || max_len < 0 ||
        (reinterpret_cast<uintptr_t>(cache_len) & 3u))
        return BD_ERR_INVALID_ARG;
    bd::bd_cache_crop_kernel<<<(B + 255) / 256, 256, 0, stream>>>(cache_len, B, max_len);
    return cudaGetLastError() == cudaSuccess ? BD_OK : BD_ERR_CUDA;
}

size_t bd_sprint_workspace_bytes(int B, int S_cap)
{
    if (B <= 0 || S_cap <= 0)
        return 0;
    return 2 * round256((size_t)B * S_cap * sizeof(double));
}

bd_status bd_sprint_prune(const void *k_cache, const void *v_cache,
                          const int32_t *cache_len, const float *conf,
                          const uint8_t *modality, float alpha,
                          float keep_text, float keep_image, void *k_out,
                          void *v_out, int32_t *kept, int32_t *new_len,
                          double *score, int B, int Hkv, int d, int S_cap,
                          cudaStream_t stream, void *workspace,
                          size_t workspace_bytes)
{
    if (!k_cache || !v_cache || !cache_len || !conf || !modality || !k_out ||
        !v_out || !kept || !new_len || !workspace)
        return BD_ERR_INVALID_ARG;
    if (B <= 0 || Hkv <= 0 || d <= 0 || S_cap <= 0)
        return BD_ERR_INVALID_ARG;
    if (!(alpha >= 0.f && alpha <= 1.f) || !(keep_text >= 0.f && keep_text <= 1.f) ||
        !(keep_image >= 0.f && keep_image <= 1.f))
        return BD_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_out) ||
        !aligned16(v_out) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        ((reinterpret_cast<uintptr_t>(cache_len) | reinterpret_cast<uintptr_t>(conf) |
          reinterpret_cast<uintptr_t>(kept) | reinterpret_cast<uintptr_t>(new_len)) & 3u) ||
        (score && (reinterpret_cast<uintptr_t>(score) & 7u)))
        return BD_ERR_INVALID_ARG;
    if (k_out == k_cache || v_out == v_cache || k_out == v_cache || v_out == k_cache)
        return BD_ERR_INVALID_ARG;
    if (workspace_bytes < bd_sprint_workspace_bytes(B, S_cap))
        return BD_ERR_INVALID_ARG;
    if (!supported_d(d))
        return BD_ERR_UNSUPPORTED;
    // the select kernel holds at most 64 positions per thread
    if (S_cap > 64 * bd::kSelThreads || B > 65535)
        return BD_ERR_UNSUPPORTED;
    double *norm = static_cast<double *>(workspace);
    double *sc = score ? score
                       : reinterpret_cast<double *>(static_cast<char *>(workspace) +
                                                    round256((size_t)B * S_cap * sizeof(double)));
    dim3 gn((S_cap + 8 * bd::kNormPos - 1) / (8 * bd::kNormPos), B);
    bd::bd_sprint_norm_kernel<<<gn, 256, 0, stream>>>(static_cast<const bf16 *>(k_cache),
                                                      cache_len, norm, Hkv, d, S_cap);
    if (cudaGetLastError() != cudaSuccess)
        return BD_ERR_CUDA;
    // a thread's run of the prefix fits its registers up to 16 positions
    if (S_cap <= 16 * bd::kSelThreads)
        bd::bd_sprint_select_kernel<16><<<B, bd::kSelThreads, 0, stream>>>(
            norm, cache_len, conf, modality, (double)alpha, (double)keep_text,
            (double)keep_image, sc, kept, new_len, S_cap);
    else
        bd::bd_sprint_select_kernel<0><<<B, bd::kSelThreads, 0, stream>>>(
            norm, cache_len, conf, modality, (double)alpha, (double)keep_text,
            (double)keep_image, sc, kept, new_len, S_cap);
    if (cudaGetLastError() != cudaSuccess)
        return BD_ERR_CUDA;
    bd::bd_sprint_compact_kernel<<<dim3((S_cap + 7) / 8, B), 256, 0, stream>>>(
        static_cast<const bf16 *>(k_cache), static_cast<const bf16 *>(v_cache), kept, new_len,
        static_cast<bf16 *>(k_out), static_cast<bf16 *>(v_out), Hkv, d, S_cap);
    return cudaGetLastError() == cudaSuccess ? BD_OK : BD_ERR_CUDA;
}

bd_status bd_attn_debug_inject_fault(int kind)
{
    if (kind != 0 && kind != 1)
        return BD_ERR_INVALID_ARG;
    return cudaMemcpyToSymbol(bd::g_fault_skip_k, &kind, sizeof kind) == cudaSuccess
               ? BD_OK
               : BD_ERR_CUDA;
}

int bd_attn_debug_fwd_kernel(int Hq, int Hkv, int d)
{
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || !supported_d(d))
        return -1;
    return ((Hq / Hkv) % 2 == 0 && pair_kernel_usable(d)) ? 2 : 1;
}

bd_status bd_attn_debug_set_grid(int ctas)
{
    if (ctas < 0 || ctas > kMaxGrid)
        return BD_ERR_INVALID_ARG;
    g_grid_cap.store(ctas);
    return BD_OK;
}

bd_status bd_attn_debug_set_chunk(int groups)
{
    if (groups < 0)
        return BD_ERR_INVALID_ARG;
    g_chunk_fixed.store(groups);
    return BD_OK;
}

bd_status bd_attn_debug_reset_sched(void)
{
    unsigned int zero[bd::kSchedSlots] = {};
    if (cudaDeviceSynchronize() != cudaSuccess)
        return BD_ERR_CUDA;
    return (cudaMemcpyToSymbol(bd::g_sched_next, zero, sizeof zero) == cudaSuccess &&
            cudaMemcpyToSymbol(bd::g_sched_done, zero, sizeof zero) == cudaSuccess &&
            cudaMemcpyToSymbol(bd::g_sched_claim, zero, sizeof zero) == cudaSuccess)
               ? BD_OK
               : BD_ERR_CUDA;
}

bd_status bd_attn_get_device_status(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return BD_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, bd::g_status_word, sizeof word) !=
        cudaSuccess)
        return BD_ERR_CUDA;
    if (word != 0 &&
        cudaMemcpyToSymbol(bd::g_status_word, &zero, sizeof zero) != cudaSuccess)
        return BD_ERR_CUDA;
    return word ? BD_ERR_DEVICE_TIMEOUT : BD_OK;
}

} // extern "C"

// ---------------------------------------------------------------------------
// Block decode without allocation: the split-KV scratch is this fixed array
// in the library's device memory.  Host code must not use the array's name as
// an address (on the host it is only a stand-in); the device address is
// looked up once per device with cudaGetSymbolAddress and passed to the
// kernels.

static __device__ __align__(256) unsigned char
    g_noalloc_scratch[BD_ATTN_NOALLOC_SCRATCH_BYTES];
// the decode scratch is the same for every size (decode_plan); it fits
static_assert(2 * kMaxGrid * bd::kTcM * bd::kTcD * sizeof(float) +
                      2 * kMaxGrid * bd::kTcM * sizeof(float) + kMaxGrid * sizeof(int4) +
                      3 * 256 <=
                  BD_ATTN_NOALLOC_SCRATCH_BYTES,
              "the fixed no-alloc array must hold the decode scratch");

namespace {

struct NoallocScratch {
    std::mutex mu;
    void *addr[64] = {};
};
NoallocScratch g_noalloc;

// Device address of g_noalloc_scratch on the current device (looked up on
// the first call for that device, with that device current).
bd_status noalloc_scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return BD_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc.mu);
    if (!g_noalloc.addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return BD_ERR_CUDA;
        g_noalloc.addr[dev] = p;
    }
    *out = g_noalloc.addr[dev];
    return BD_OK;
}

} // namespace

extern "C" bd_status bd_attn_decode_noalloc(
    const void *q_blk, const void *k_cache, const void *v_cache,
    const int32_t *cache_len, void *out, float *lse, int B, int Hq, int Hkv,
    int b, int d, int intra_block_mode, cudaStream_t stream, int S_cap)
{
    DecodePlan pl;
    bd_status st = decode_validate(q_blk, k_cache, v_cache, cache_len, out,
                                   lse, B, Hq, Hkv, b, d, intra_block_mode,
                                   S_cap, pl);
    if (st != BD_OK)
        return st;
    if (pl.total_bytes > (size_t)BD_ATTN_NOALLOC_SCRATCH_BYTES)
        return BD_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    st = noalloc_scratch_address(&scratch);
    if (st != BD_OK)
        return st;
    return decode_launch(q_blk, k_cache, v_cache, cache_len, out, lse, B, Hq,
                         Hkv, b, d, intra_block_mode, stream, S_cap, scratch,
                         pl);
}

#ifdef BD_TC_TRACE
// Debug builds only: point the tensor-core kernels' progress trace at a
// host-mapped buffer of 8 words per CTA (NULL disables it).
extern "C" __attribute__((visibility("default"))) int
bd_debug_set_trace(void *buf)
{
    uint32_t *p = static_cast<uint32_t *>(buf);
    return cudaMemcpyToSymbol(bd::g_tc_trace, &p, sizeof p) == cudaSuccess ? 0 : 1;
}
#endif
