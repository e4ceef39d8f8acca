// KV-cache kernels of block decoding (sm_100a): accepting a speculated
// block, appending it to the cache, cropping the cache, and sparse prefix
// retention (SPRINT).
//
//  - Speculative accept / append / crop: "Nemotron-Labs-Diffusion-8B-Base 3x
//    decoding speed-up", section 2 "Linear Speculative Decoding" (draft a
//    block with bidirectional attention, validate it with causal attention,
//    accept the longest matching prefix, update the KV cache) and section
//    "KV cache strategy" (crop the cache to a maximum length).
//  - Sparse prefix retention: "LLaDA2.0-Uni", section "SPRINT: training-free
//    inference acceleration", paragraph "Sparse Prefix Retention": once per
//    block, score every prefix position by s_i = alpha * I_i + (1 - alpha) *
//    c_i, I_i = |k_i|_2 / mean_j |k_j|_2, and keep each modality's best
//    fraction (images 0.8, text 1.0 on the page).
//
// Layouts as in the attention kernels: caches [B, Hkv, S_cap, d] bf16,
// cache_len [B] int32 on the device.  All of it is HBM- or latency-bound:
// 16-byte vector copies, fp64 only for the SPRINT scores (so the kept set
// is decided in double precision).
#pragma once

#include "bd_common.cuh"

namespace bd {

// ---------------------------------------------------------------------------
// speculative decoding: accepted length, append, crop

// n_accept[i] = length of the longest prefix of block positions j on which
// draft[i][j] == target[i][j].  One warp per sequence.
__global__ void __launch_bounds__(256)
    bd_spec_accept_kernel(const int32_t *draft, const int32_t *target,
                          int32_t *n_accept, int B, int b)
{
    const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (i >= B)
        return;
    const int32_t *dr = draft + (size_t)i * b;
    const int32_t *tg = target + (size_t)i * b;
    int n = b;
    for (int j0 = 0; j0 < b; j0 += 32) {
        const int j = j0 + lane;
        const bool differ = j < b && dr[j] != tg[j];
        const unsigned m = __ballot_sync(0xffffffffu, differ);
        if (m) {
            n = j0 + __ffs(m) - 1;
            break;
        }
    }
    if (lane == 0)
        n_accept[i] = n;
}

// Appends rows 0 .. n_new[i]-1 of the block K/V ([B, Hkv, b, d]; NULL: the
// rows already sit at cache positions cache_len[i] ..) and advances
// cache_len[i].  One CTA per sequence, so the length is updated after every
// copy of that sequence has read it.  An out-of-range n_new or length leaves
// the sequence untouched and records DEV_BAD_CACHE_LEN.
__global__ void __launch_bounds__(512)
    bd_cache_append_kernel(bf16 *k_cache, bf16 *v_cache, int32_t *cache_len,
                           const bf16 *k_new, const bf16 *v_new,
                           const int32_t *n_new, int Hkv, int b, int d,
                           int S_cap)
{
    const int i = blockIdx.x;
    const int len = cache_len[i];
    const int n = n_new[i];
    if (n < 0 || n > b || len < 0 || (long long)len + n > S_cap) {
        if (threadIdx.x == 0)
            raise_device_code(DEV_BAD_CACHE_LEN);
        return;
    }
    if (k_new != nullptr) {
        const int vec_per_row = d / 8; // 16-byte vectors
        const long long total = (long long)Hkv * n * vec_per_row;
        for (long long e = threadIdx.x; e < total; e += blockDim.x) {
            const int c = (int)(e % vec_per_row);
            const long long rr = e / vec_per_row;
            const int r = (int)(rr % n), h = (int)(rr / n);
            const size_t src = (((size_t)i * Hkv + h) * b + r) * d + (size_t)c * 8;
            const size_t dst = (((size_t)i * Hkv + h) * S_cap + len + r) * d + (size_t)c * 8;
            reinterpret_cast<uint4 *>(k_cache + dst)[0] =
                reinterpret_cast<const uint4 *>(k_new + src)[0];
            reinterpret_cast<uint4 *>(v_cache + dst)[0] =
                reinterpret_cast<const uint4 *>(v_new + src)[0];
        }
    }
    __syncthreads();
    if (threadIdx.x == 0)
        cache_len[i] = len + n;
}

// cache_len[i] = min(cache_len[i], max_len).
__global__ void __launch_bounds__(256)
    bd_cache_crop_kernel(int32_t *cache_len, int B, int max_len)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < B)
        cache_len[i] = min(cache_len[i], max_len);
}

// ---------------------------------------------------------------------------
// sparse prefix retention

// |k_p|_2 over all kv-heads and dims of position p, for p < cache_len[i]:
// norm[i][p] in fp64.  A warp takes kNormPos consecutive positions, lane l
// reading 16-byte pieces of their Hkv rows (each row contiguous, two rows per
// warp load); all of a warp's loads are issued before the sums.
constexpr int kNormPos = 4;

__global__ void __launch_bounds__(256)
    bd_sprint_norm_kernel(const bf16 *k_cache, const int32_t *cache_len,
                          double *norm, int Hkv, int d, int S_cap)
{
    const int i = blockIdx.y;
    const int pbase = (blockIdx.x * 8 + (threadIdx.x >> 5)) * kNormPos;
    const int lane = threadIdx.x & 31;
    const int len = cache_len[i];
    if (pbase >= len || len > S_cap)
        return;
    const int vec_per_row = d / 8;
    const int nvec = Hkv * vec_per_row; // multiple of 4 (d >= 32)
    double ss[kNormPos];
#pragma unroll
    for (int q = 0; q < kNormPos; ++q)
        ss[q] = 0.0;
    for (int e0 = 0; e0 < nvec; e0 += 32) {
        const int e = e0 + lane;
        uint4 x[kNormPos];
#pragma unroll
        for (int q = 0; q < kNormPos; ++q) {
            const int p = pbase + q;
            x[q] = make_uint4(0, 0, 0, 0);
            if (e < nvec && p < len) {
                const int h = e / vec_per_row, c = e % vec_per_row;
                x[q] = *reinterpret_cast<const uint4 *>(
                    k_cache + (((size_t)i * Hkv + h) * S_cap + p) * d + (size_t)c * 8);
            }
        }
#pragma unroll
        for (int q = 0; q < kNormPos; ++q) {
            const uint32_t w[4] = {x[q].x, x[q].y, x[q].z, x[q].w};
#pragma unroll
            for (int t4 = 0; t4 < 4; ++t4) {
                // bf16 squares are exact in fp64
                const double lo = (double)__uint_as_float(w[t4] << 16);
                const double hi = (double)__uint_as_float(w[t4] & 0xffff0000u);
                ss[q] = fma(lo, lo, ss[q]);
                ss[q] = fma(hi, hi, ss[q]);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < kNormPos; ++q) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            ss[q] += __shfl_xor_sync(0xffffffffu, ss[q], o);
        if (lane == 0 && pbase + q < len)
            norm[(size_t)i * S_cap + pbase + q] = sqrt(ss[q]);
    }
}

constexpr int kSelThreads = 1024;

// Order-preserving map of a double onto uint64 (larger value -> larger key).
__device__ __forceinline__ unsigned long long dkey(double x)
{
    const unsigned long long u = (unsigned long long)__double_as_longlong(x);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

template <typename T> __device__ T block_sum(T v, T *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0)
        red[w] = v;
    __syncthreads();
    T tot = 0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k)
        tot += red[k];
    return tot;
}

// Exclusive prefix sum of one int per thread over the block (in thread
// order); returns the thread's offset and writes the total.
__device__ int block_scan_excl(int v, int *red, int &total)
{
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o)
            x += y;
    }
    __syncthreads();
    if (lane == 31)
        red[w] = x;
    __syncthreads();
    int base = 0, tot = 0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) {
        if (k < w)
            base += red[k];
        tot += red[k];
    }
    total = tot;
    return base + x - v;
}

// Scores, per-modality selection and the kept list of one sequence per CTA.
//   score[i][p] = alpha * norm_p / mean + (1 - alpha) * conf[i][p] (fp64),
//   per modality m (0 text, else image) with n_m prefix positions keep the
//   floor(r_m n_m + 1/2) best (higher score, then lower position),
//   kept[i][0 .. new_len-1] = kept positions in increasing order, then -1.
// The threshold of each modality is found by an 8-pass radix select (8 bits
// per pass) over the score keys; positions are visited in contiguous
// per-thread runs so that the final scan keeps position order.  With
// PER > 0 a thread's run (at most PER positions) is held in registers;
// PER = 0 reads it from memory on every pass (long prefixes).
template <int PER>
__global__ void __launch_bounds__(kSelThreads)
    bd_sprint_select_kernel(const double *norm, const int32_t *cache_len,
                            const float *conf, const uint8_t *modality,
                            double alpha, double keep_text, double keep_image,
                            double *score, int32_t *kept, int32_t *new_len,
                            int S_cap)
{
    __shared__ double red_d[32];
    __shared__ int red_i[32];
    __shared__ unsigned int hist[512];
    __shared__ unsigned long long s_prefix[2];
    __shared__ int s_need[2], s_want[2];
    const int i = blockIdx.x;
    const int len = cache_len[i];
    const int tid = threadIdx.x;
    const size_t row = (size_t)i * S_cap;
    if (len < 0 || len > S_cap) {
        if (tid == 0) {
            raise_device_code(DEV_BAD_CACHE_LEN);
            new_len[i] = 0;
        }
        for (int p = tid; p < S_cap; p += blockDim.x)
            kept[row + p] = -1;
        return;
    }
    // this thread's contiguous run of positions [p0, p1)
    const int per = (len + blockDim.x - 1) / blockDim.x;
    const int p0 = min(len, tid * per), p1 = min(len, p0 + per);
    const int cnt = p1 - p0;

    double part = 0.0;
    for (int p = p0; p < p1; ++p)
        part += norm[row + p];
    const double mean = block_sum(part, red_d) / (double)max(len, 1);
    // run cache: score key and modality bit of each position of the run;
    // every loop over the run is unrolled to RMAX with an early exit, so
    // the cache stays in registers
    constexpr int RMAX = PER > 0 ? PER : 64;
    constexpr int R = PER > 0 ? PER : 1;
    unsigned long long rk[R];
    uint64_t rm = 0;
    int nimg = 0;
#pragma unroll
    for (int u = 0; u < RMAX; ++u) {
        if (u >= cnt)
            break;
        const int p = p0 + u;
        // separate roundings, no fused multiply-add: the same arithmetic as
        // the plain definition, so equal inputs give equal scores
        const double inorm = mean > 0.0 ? __ddiv_rn(norm[row + p], mean) : 0.0;
        const double sc = __dadd_rn(__dmul_rn(alpha, inorm),
                                    __dmul_rn(__dadd_rn(1.0, -alpha), (double)conf[row + p]));
        score[row + p] = sc;
        const int m = modality[row + p] != 0;
        nimg += m;
        if (PER > 0) {
            rk[PER > 0 ? u : 0] = dkey(sc);
            rm |= (uint64_t)m << u;
        }
    }
    // key and modality of run position u
    auto key_at = [&](int u, int &m) -> unsigned long long {
        if (PER > 0) {
            m = (int)((rm >> u) & 1u);
            return rk[PER > 0 ? u : 0];
        }
        m = modality[row + p0 + u] != 0;
        return dkey(score[row + p0 + u]);
    };
    {
        const int n_img = block_sum(nimg, red_i);
        if (tid == 0) {
            const int n_m[2] = {len - n_img, n_img};
            for (int m = 0; m < 2; ++m) {
                const double r = m == 0 ? keep_text : keep_image;
                long long want = (long long)floor(r * (double)n_m[m] + 0.5);
                want = max(0LL, min(want, (long long)n_m[m]));
                s_want[m] = (int)want;
                s_need[m] = (int)want; // rank still to find below the prefix
                s_prefix[m] = 0;
            }
        }
        __syncthreads();
    }
    // kept flags live in the kept row itself until the final compaction:
    // 1 = kept, 0 = dropped.  Both modalities are selected together, one
    // 256-bin histogram per modality.
    for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int k = tid; k < 512; k += blockDim.x)
            hist[k] = 0;
        __syncthreads();
        const unsigned long long hmask = pass == 0 ? 0ull : (~0ull << (shift + 8));
        const unsigned long long pre0 = s_prefix[0], pre1 = s_prefix[1];
#pragma unroll
        for (int u = 0; u < RMAX; ++u) {
            if (u >= cnt)
                break;
            int m;
            const unsigned long long key = key_at(u, m);
            if ((key & hmask) == (m ? pre1 : pre0))
                atomicAdd(&hist[m * 256 + ((key >> shift) & 255)], 1u);
        }
        __syncthreads();
        // warp m finds the digit of modality m: lane l owns the 8 digits
        // 255 - 8 l .. 248 - 8 l, scanned from the top
        const int w = tid >> 5, lane = tid & 31;
        if (w < 2 && s_want[w] > 0) {
            const unsigned int *hm = hist + w * 256;
            int sum = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                sum += (int)hm[255 - 8 * lane - u];
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += y;
            }
            const int need = s_need[w];
            const unsigned int hit = __ballot_sync(0xffffffffu, incl >= need);
            // need >= 1 and the modality's candidates number at least need,
            // so some lane holds the target
            const int tl = __ffs(hit) - 1;
            if (lane == tl) {
                int rem = need - (incl - sum);
                int dgt = 255 - 8 * lane;
                for (int u = 0; u < 7; ++u, --dgt) {
                    if ((int)hm[dgt] >= rem)
                        break;
                    rem -= (int)hm[dgt];
                }
                s_prefix[w] |= (unsigned long long)dgt << shift;
                s_need[w] = rem;
            }
        }
        __syncthreads();
    }
    // keys above a modality's threshold are kept; of the keys equal to it,
    // its s_need lowest positions
    const unsigned long long thr0 = s_prefix[0], thr1 = s_prefix[1];
    const bool any0 = s_want[0] > 0, any1 = s_want[1] > 0;
    int eq[2] = {0, 0};
#pragma unroll
    for (int u = 0; u < RMAX; ++u) {
        if (u >= cnt)
            break;
        int m;
        const unsigned long long key = key_at(u, m);
        eq[m] += (m ? any1 : any0) && key == (m ? thr1 : thr0);
    }
    int tot0, tot1;
    int before0 = block_scan_excl(eq[0], red_i, tot0);
    int before1 = block_scan_excl(eq[1], red_i, tot1);
    const int need0 = any0 ? s_need[0] : 0, need1 = any1 ? s_need[1] : 0;
    int mine = 0;
    uint64_t keepbits = 0;
#pragma unroll
    for (int u = 0; u < RMAX; ++u) {
        if (u >= cnt)
            break;
        int m;
        const unsigned long long key = key_at(u, m);
        const unsigned long long thr = m ? thr1 : thr0;
        int keep = 0;
        if (m ? any1 : any0) {
            if (key > thr)
                keep = 1;
            else if (key == thr)
                keep = m ? (before1++ < need1) : (before0++ < need0);
        }
        if (PER > 0)
            keepbits |= (uint64_t)keep << u;
        else
            kept[row + p0 + u] = keep;
        mine += keep;
    }

    // stable compaction of the kept positions
    int total;
    int dst = block_scan_excl(mine, red_i, total);
    if (PER == 0) {
        // the flags of this thread's run are in memory: read them before
        // any thread overwrites them with positions (a thread's
        // destinations reach into the runs of threads before it only)
        for (int u = 0; u < cnt; ++u)
            keepbits |= (uint64_t)kept[row + p0 + u] << u;
        __syncthreads();
    }
    for (int u = 0; u < cnt; ++u)
        if ((keepbits >> u) & 1u)
            kept[row + dst++] = p0 + u;
    __syncthreads();
    for (int p = total + tid; p < S_cap; p += blockDim.x)
        kept[row + p] = -1;
    if (tid == 0)
        new_len[i] = total;
}

// k_out/v_out rows 0 .. new_len[i]-1 = k_cache/v_cache rows kept[i][0 ..]
// for every kv-head.  Grid (S_cap / 8 tiles, B); one warp per destination
// row of all heads, 16-byte vectors.
__global__ void __launch_bounds__(256)
    bd_sprint_compact_kernel(const bf16 *k_cache, const bf16 *v_cache,
                             const int32_t *kept, const int32_t *new_len,
                             bf16 *k_out, bf16 *v_out, int Hkv, int d,
                             int S_cap)
{
    const int i = blockIdx.y;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= new_len[i])
        return;
    const int src = kept[(size_t)i * S_cap + t];
    if (src < 0 || src >= S_cap) { // cannot happen after the select kernel
        if (lane == 0)
            raise_device_code(DEV_BAD_CACHE_LEN);
        return;
    }
    const int vec_per_row = d / 8;
    const int nvec = Hkv * vec_per_row;
    for (int e = lane; e < nvec; e += 32) {
        const int h = e / vec_per_row, c = e % vec_per_row;
        const size_t hb = ((size_t)i * Hkv + h) * S_cap;
        const size_t so = (hb + src) * d + (size_t)c * 8;
        const size_t dof = (hb + t) * d + (size_t)c * 8;
        reinterpret_cast<uint4 *>(k_out + dof)[0] = reinterpret_cast<const uint4 *>(k_cache + so)[0];
        reinterpret_cast<uint4 *>(v_out + dof)[0] = reinterpret_cast<const uint4 *>(v_cache + so)[0];
    }
}

} // namespace bd
