// Block-diffusion attention on the warp-level mma.sync tensor path
// (m16n8k16, bf16 in, fp32 accumulate), FlashAttention-2 style.
//
// One CTA = 4 warps = a 64-row query tile; each warp owns 16 rows.  K/V tiles
// of 64 keys stream through a double-buffered, XOR-swizzled shared-memory
// ring fed by 16-byte cp.async; S = QK^T and O += PV run on mma.sync; the
// online softmax lives in registers.  Used for the split-KV block decode at
// head dim 32 (the training/prefill form runs on the tcgen05 kernels at every
// head dim, and so does the decode at 64 and 128).
//
// Every query row's visible key set is two intervals [a0,a1) U [a2,a3):
//   training/prefill, noisy row of block k : [k b, k b + b) U [L, L + k b)
//   training/prefill, clean row of block k : {}             U [L, L + (k+1) b)
//   decode row j of a block after n cached : [0, n + b)   (bidirectional)
//                                            [0, n + j + 1) (causal)
// which is the three-part mask M_BD / M_OBC / M_BC of "Nemotron-Labs-
// Diffusion-8B-Base 3x decoding speed-up", section 1 "Block Diffusion
// Attention", and the draft/verify attention of its section 2.
#pragma once

#include "bd_common.cuh"

namespace bd {

typedef __nv_bfloat16 bf16;

struct MmaParams {
    const bf16 *q, *k, *v;
    bf16 *out;
    float *lse;
    float *part_o;   // decode: [nsplit][B*Hq*b][d] fp32 partial outputs
    float *part_lse; // decode: [nsplit][B*Hq*b] partial lse (natural log)
    const int32_t *cache_len;
    int B, Hq, Hkv, L, b;
    int nkeys;   // key rows per kv-head in memory: 2L (fwd) or S_cap (decode)
    int mode;    // decode: 0 bidirectional, 1 causal inside the block
    int chunk;   // decode: keys per split
    int nsplit;  // decode: splits per (batch, kv-head)
    float scale_log2; // softmax scale * log2(e)
};

constexpr int kMmaBM = 64;
constexpr int kMmaBN = 64;
constexpr int kMmaThreads = 128;

template <int D> constexpr int mma_smem_bytes()
{
    return 5 * kMmaBM * D * 2; // Q + 2 x K + 2 x V tiles
}

// Swizzled element offset of (row r, column col) in a 64 x D bf16 tile; the
// 16-byte chunk index is XORed with low row bits so that ldmatrix of 8
// consecutive rows hits 8 distinct bank groups.
template <int D> __device__ __forceinline__ int soff(int r, int col)
{
    int c = col >> 3;
    int sw = (D == 32) ? (c ^ ((r >> 1) & 3)) : (c ^ (r & 7));
    return r * D + (sw << 3) + (col & 7);
}

// Async copy of rows [row0, row0 + nvalid) of a row-major [*, D] bf16 tensor
// into a 64-row swizzled tile; rows >= nvalid are zero-filled.
template <int D>
__device__ __forceinline__ void load_tile(bf16 *s, const bf16 *g, int row0,
                                          int nvalid)
{
    constexpr int CPR = D / 8;
    for (int i = threadIdx.x; i < kMmaBM * CPR; i += kMmaThreads) {
        int r = i / CPR, c = i % CPR;
        bool ok = r < nvalid;
        const bf16 *src = ok ? g + (size_t)(row0 + r) * D + c * 8 : g;
        cp_async16(s + soff<D>(r, c * 8), src, ok ? 16 : 0);
    }
}

struct Span {
    int a0, a1, a2, a3;
};

__device__ __forceinline__ bool span_has(const Span &s, int c)
{
    return (c >= s.a0 && c < s.a1) || (c >= s.a2 && c < s.a3);
}

// Per-CTA work description.
struct Plan {
    int nrows;          // valid rows in the tile (<= 64)
    int lo[2], hi[2];   // key ranges to visit
    int flo[2], fhi[2]; // keys in [flo, fhi) are visible to every row
    // decode only
    int len, row0, gbase; // cache length, first local row, global row base
    int split;
};

__device__ __forceinline__ Span fwd_span(int L, int b, int r)
{
    Span s;
    if (r < L) {
        int kb = r / b;
        s.a0 = kb * b; s.a1 = kb * b + b; s.a2 = L; s.a3 = L + kb * b;
    } else {
        int kb = (r - L) / b;
        s.a0 = 0; s.a1 = 0; s.a2 = L; s.a3 = L + (kb + 1) * b;
    }
    return s;
}

__device__ __forceinline__ Span decode_span(const MmaParams &p, const Plan &pl,
                                            int rloc)
{
    int j = (pl.row0 + rloc) % p.b;
    int hi = pl.len + (p.mode == 0 ? p.b : p.mode == 1 ? j + 1 : 0);
    int s0 = pl.split * p.chunk;
    Span s;
    s.a0 = s0; s.a1 = min(hi, s0 + p.chunk); s.a2 = 0; s.a3 = 0;
    return s;
}

// the CTA's (batch, kv-head, split, row tile); false if it has no keys
__device__ __forceinline__ bool make_plan(const MmaParams &p, Plan &pl)
{
    const int unit = blockIdx.z; // batch * Hkv + kv-head
    const int bi = unit / p.Hkv, g = unit % p.Hkv;
    const int group = p.Hq / p.Hkv;
    const int len = p.cache_len[bi];
    const int s = blockIdx.x;
    const int own = p.mode == 2 ? 0 : p.b; // keys past the prefix
    if (len < 0 || (long long)len + own > p.nkeys)
        return false; // reported by the combine kernel
    const int total = len + own;
    if (s * p.chunk >= total)
        return false;
    pl.len = len;
    pl.split = s;
    pl.row0 = blockIdx.y * kMmaBM;
    pl.nrows = min(kMmaBM, group * p.b - pl.row0);
    pl.gbase = (bi * p.Hq + g * group) * p.b; // global row of local row 0
    const int s0 = s * p.chunk, s1 = min(total, s0 + p.chunk);
    pl.lo[0] = s0; pl.hi[0] = s1;
    pl.lo[1] = 0; pl.hi[1] = 0;
    pl.flo[0] = s0;
    pl.fhi[0] = min(s1, len + (p.mode == 0 ? p.b : 0));
    pl.flo[1] = 0; pl.fhi[1] = 0;
    return true;
}

template <int D>
__global__ void __launch_bounds__(kMmaThreads)
    bd_mma_attn_kernel(const MmaParams p)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    bf16 *sQ = reinterpret_cast<bf16 *>(smem_raw);
    bf16 *sK = sQ + kMmaBM * D;
    bf16 *sV = sK + 2 * kMmaBM * D;

    Plan pl;
    if (!make_plan(p, pl))
        return;

    const int unit = blockIdx.z;
    const bf16 *qsrc = p.q + ((size_t)pl.gbase + pl.row0) * D;
    const bf16 *kbase = p.k + (size_t)unit * p.nkeys * D;
    const bf16 *vbase = p.v + (size_t)unit * p.nkeys * D;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;

    // spans of the two rows this thread holds (warp*16 + gq, +8)
    Span sp[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        int rl = min(warp * 16 + gq + 8 * i, pl.nrows - 1);
        sp[i] = decode_span(p, pl, rl);
    }

    // key tiles: range 0 then range 1
    const int n0 = pl.hi[0] > pl.lo[0] ? (pl.hi[0] - pl.lo[0] + kMmaBN - 1) / kMmaBN : 0;
    const int n1 = pl.hi[1] > pl.lo[1] ? (pl.hi[1] - pl.lo[1] + kMmaBN - 1) / kMmaBN : 0;
    const int nt = n0 + n1;

    load_tile<D>(sQ, qsrc, 0, pl.nrows);
    cp_async_commit();
    auto tile_of = [&](int it, int &ks, int &rg) {
        rg = it < n0 ? 0 : 1;
        ks = pl.lo[rg] + (it - (rg ? n0 : 0)) * kMmaBN;
    };
    if (nt > 0) {
        int ks, rg;
        tile_of(0, ks, rg);
        load_tile<D>(sK, kbase, ks, pl.hi[rg] - ks);
        load_tile<D>(sV, vbase, ks, pl.hi[rg] - ks);
    }
    cp_async_commit();

    uint32_t qa[D / 16][4];
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
        o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY};
    float l[2] = {0.f, 0.f};

    for (int it = 0; it < nt; ++it) {
        if (it + 1 < nt) {
            int ks, rg;
            tile_of(it + 1, ks, rg);
            int buf = (it + 1) & 1;
            load_tile<D>(sK + buf * kMmaBM * D, kbase, ks, pl.hi[rg] - ks);
            load_tile<D>(sV + buf * kMmaBM * D, vbase, ks, pl.hi[rg] - ks);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (it == 0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                ldmatrix_x4(qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3],
                            sQ + soff<D>(warp * 16 + (lane & 15),
                                         kk * 16 + (lane >> 4) * 8));
        }
        const bf16 *tK = sK + (it & 1) * kMmaBM * D;
        const bf16 *tV = sV + (it & 1) * kMmaBM * D;
        int ks, rg;
        tile_of(it, ks, rg);
        const int khi = pl.hi[rg];

        float s[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                int mi = lane >> 3;
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(b0, b1, b2, b3,
                            tK + soff<D>(np * 16 + (mi >> 1) * 8 + (lane & 7),
                                         kk * 16 + (mi & 1) * 8));
                mma_bf16_16816(s[2 * np], qa[kk], b0, b1);
                mma_bf16_16816(s[2 * np + 1], qa[kk], b2, b3);
            }
        }

        // scale into the log2 domain; mask unless the whole tile is visible
        const bool full = ks >= pl.flo[rg] && ks + kMmaBN <= pl.fhi[rg] &&
                          ks + kMmaBN <= khi;
#pragma unroll
        for (int nt8 = 0; nt8 < 8; ++nt8) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float x = s[nt8][e] * p.scale_log2;
                if (!full) {
                    int c = ks + nt8 * 8 + 2 * tq + (e & 1);
                    if (!(c < khi && span_has(sp[e >> 1], c)))
                        x = -INFINITY;
                }
                s[nt8][e] = x;
            }
        }
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt8 = 0; nt8 < 8; ++nt8) {
            mx[0] = fmaxf(mx[0], fmaxf(s[nt8][0], s[nt8][1]));
            mx[1] = fmaxf(mx[1], fmaxf(s[nt8][2], s[nt8][3]));
        }
        float corr[2], muse[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
            float mn = fmaxf(m[i], mx[i]);
            muse[i] = (mn == -INFINITY) ? 0.f : mn;
            corr[i] = ex2(m[i] - muse[i]);
            m[i] = mn;
        }
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int nt8 = 0; nt8 < 8; ++nt8) {
            s[nt8][0] = ex2(s[nt8][0] - muse[0]);
            s[nt8][1] = ex2(s[nt8][1] - muse[0]);
            s[nt8][2] = ex2(s[nt8][2] - muse[1]);
            s[nt8][3] = ex2(s[nt8][3] - muse[1]);
            rs[0] += s[nt8][0] + s[nt8][1];
            rs[1] += s[nt8][2] + s[nt8][3];
        }
        l[0] = l[0] * corr[0] + rs[0];
        l[1] = l[1] * corr[1] + rs[1];
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            o[i][0] *= corr[0]; o[i][1] *= corr[0];
            o[i][2] *= corr[1]; o[i][3] *= corr[1];
        }
#pragma unroll
        for (int kk2 = 0; kk2 < 4; ++kk2) {
            uint32_t pa[4];
            pa[0] = pack_bf16x2(s[2 * kk2][0], s[2 * kk2][1]);
            pa[1] = pack_bf16x2(s[2 * kk2][2], s[2 * kk2][3]);
            pa[2] = pack_bf16x2(s[2 * kk2 + 1][0], s[2 * kk2 + 1][1]);
            pa[3] = pack_bf16x2(s[2 * kk2 + 1][2], s[2 * kk2 + 1][3]);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                int mi = lane >> 3;
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(b0, b1, b2, b3,
                                  tV + soff<D>(kk2 * 16 + (mi & 1) * 8 + (lane & 7),
                                               dp * 16 + (mi >> 1) * 8));
                mma_bf16_16816(o[2 * dp], pa, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
            }
        }
        __syncthreads();
    }

    // epilogue
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        l[i] += __shfl_xor_sync(0xffffffffu, l[i], 1);
        l[i] += __shfl_xor_sync(0xffffffffu, l[i], 2);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int rl = warp * 16 + gq + 8 * i;
        if (rl >= pl.nrows)
            continue;
        const float inv = l[i] > 0.f ? 1.f / l[i] : 0.f;
        const float lse = l[i] > 0.f ? (m[i] + __log2f(l[i])) * kLn2 : -INFINITY;
        const size_t rows_all = (size_t)p.B * p.Hq * p.b;
        const size_t row = (size_t)pl.gbase + pl.row0 + rl;
        float *orow = p.part_o + ((size_t)pl.split * rows_all + row) * D;
#pragma unroll
        for (int nt8 = 0; nt8 < D / 8; ++nt8) {
            float2 v2 = make_float2(o[nt8][2 * i] * inv,
                                    o[nt8][2 * i + 1] * inv);
            *reinterpret_cast<float2 *>(orow + nt8 * 8 + 2 * tq) = v2;
        }
        if (tq == 0)
            p.part_lse[(size_t)pl.split * rows_all + row] = lse;
    }
}

// Merge the per-split partial results of every decode row:
// lse = ln sum_s exp(lse_s), out = sum_s exp(lse_s - lse) o_s, over the splits
// that hold keys of that sequence.  One warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    bd_decode_combine_kernel(const MmaParams p)
{
    const int rows_all = p.B * p.Hq * p.b;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows_all)
        return;
    const int bi = row / (p.Hq * p.b);
    const int len = p.cache_len[bi];
    constexpr int PER = D / 32;
    bf16 *orow = p.out + (size_t)row * D;
    const int own = p.mode == 2 ? 0 : p.b; // keys past the prefix
    if (len < 0 || (long long)len + own > p.nkeys) {
        for (int t = 0; t < PER; ++t)
            orow[lane * PER + t] = __float2bfloat16_rn(NAN);
        if (lane == 0) {
            p.lse[row] = NAN;
            raise_device_code(DEV_BAD_CACHE_LEN);
        }
        return;
    }
    const int ns = (len + own + p.chunk - 1) / p.chunk;
    float mx = -INFINITY;
    for (int s = 0; s < ns; ++s)
        mx = fmaxf(mx, p.part_lse[(size_t)s * rows_all + row]);
    float acc[PER];
#pragma unroll
    for (int t = 0; t < PER; ++t)
        acc[t] = 0.f;
    float z = 0.f;
    if (mx != -INFINITY) {
        for (int s = 0; s < ns; ++s) {
            float ls = p.part_lse[(size_t)s * rows_all + row];
            if (ls == -INFINITY)
                continue;
            float w = ex2((ls - mx) * kLog2e);
            z += w;
            const float *src = p.part_o + ((size_t)s * rows_all + row) * D + lane * PER;
#pragma unroll
            for (int t = 0; t < PER; ++t)
                acc[t] += w * src[t];
        }
    }
    const float inv = z > 0.f ? 1.f / z : 0.f;
#pragma unroll
    for (int t = 0; t < PER; ++t)
        orow[lane * PER + t] = __float2bfloat16_rn(acc[t] * inv);
    if (lane == 0)
        p.lse[row] = z > 0.f ? mx + __logf(z) : -INFINITY;
}

} // namespace bd
