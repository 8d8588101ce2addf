// Kernels of the AWQ per-layer scale search on B200 (sm_100a).
//
//   act_stats_kernel      a_j = mean_t |X[t,j]|              (HBM-bound column reduction)
//   alpha_scales_kernel   s = a^alpha, rs = RN32(1/s)        (tiny)
//   group_params_kernel   per (alpha, row, group): sh, r, z  (one pass over W for all alphas)
//   search_pair_kernel    per alpha: sum ((W_hat - W) X^T)^2 (tcgen05 cta_group::2 / TMEM / TMA)
//   loss_reduce_kernel    per-alpha MSE and per-row sums     (deterministic, binary64)
//   best_scale_kernel     argmin over the grid + s_best
//   pack_kernel           codes / fp16 scales / fp16 zeros   (HBM-bound)
//   quant_dequant_kernel  W_hat for one s (the a3/a4 step on its own)
//   scale_table_kernel    a caller's s table checked, with RN32(1/s)  (tiny)
//   mask_columns_kernel   X with the fp16-kept channels zeroed       (HBM-bound)
//   topk_kernel           the k channels of largest statistic        (tiny)
//
// Sources (web pages): [AWQ-note] "AWQ: Activation-Aware Weight Quantization For
// On-Device LLM Compression AND Acceleration", section "Measures"; [QAS-QA]
// "Как работает quantization-aware scaling в AWQ для защиты важных весов?" §5, §6,
// §9; [GPTQ-AWQ] "GPTQ与AWQ", section "量化方法"; [AWQ-wiki] "AWQ" (French),
// "Fondements techniques".
#pragma once

#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cfloat>
#include <cstdint>

#include "awq_device.cuh"

namespace awq {

namespace cg = cooperative_groups;

// ===========================================================================
// a1. Activation statistics: a_j = RN32(RN64(sum_t |X[t,j]|) / T)
//     ([AWQ-note] "Measures"; [GPTQ-AWQ] "量化方法": X.abs().mean(dim=0)).
//
// A cluster of 8 CTAs owns a slab of 64 columns; each CTA reads every 8th
// group of 32 rows with 16-byte loads (8 threads cover one 128-byte row
// segment, 16 loads issued per batch), accumulates |x| in binary64 -- exact,
// since every fp16 value is a multiple of 2^-24 and the sums stay below 2^29,
// so the order of the additions cannot change them -- reduces its row lanes
// by warp shuffles and shared memory, and CTA 0 of the cluster sums the 8
// partial vectors through distributed shared memory.  No workspace, one launch.
// ===========================================================================
constexpr int kStatsCols = 64;
constexpr int kStatsTPR = 8;                       // threads per row segment (128 bytes)
constexpr int kStatsThreads = 256;
constexpr int kStatsWarps = kStatsThreads / 32;
constexpr int kStatsRowsPerCta = kStatsThreads / kStatsTPR;   // 32
constexpr int kStatsCluster = 8;
constexpr int kStatsUnroll = 16;                   // loads per batch

__device__ __forceinline__ void stats_accumulate(const uint4 &v, double (&acc)[8]) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(__habs2(h[e]));
        acc[2 * e] = __dadd_rn(acc[2 * e], (double)f.x);
        acc[2 * e + 1] = __dadd_rn(acc[2 * e + 1], (double)f.y);
    }
}

__global__ void __cluster_dims__(kStatsCluster, 1, 1) __launch_bounds__(kStatsThreads)
act_stats_kernel(const __half *__restrict__ X, int64_t T, int64_t K, int64_t ldx,
                 float *__restrict__ a) {
    __shared__ double red[kStatsWarps][kStatsCols];
    __shared__ double part[kStatsCols];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int slab = blockIdx.x / kStatsCluster;
    const int cc = threadIdx.x % kStatsTPR;
    const int rl = threadIdx.x / kStatsTPR;
    const int64_t col0 = (int64_t)slab * kStatsCols + cc * 8;
    const bool active = col0 < K;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;

    const int64_t rstride = (int64_t)kStatsRowsPerCta * kStatsCluster;   // 256 rows
    int64_t t = (int64_t)rank * kStatsRowsPerCta + rl;
    if (active) {
        for (; t + (kStatsUnroll - 1) * rstride < T; t += kStatsUnroll * rstride) {
            static_assert(kStatsUnroll == 16, "one batch is one ldg_stream_v4x16");
            uint4 v[kStatsUnroll];
            ldg_stream_v4x16(X + t * ldx + col0, rstride * ldx * 2, v);
#pragma unroll
            for (int u = 0; u < kStatsUnroll; ++u) stats_accumulate(v[u], acc);
        }
        for (; t < T; t += rstride) stats_accumulate(ldg_stream_v4(X + t * ldx + col0), acc);
    }
    // the warp's 4 row lanes by shuffles, the 8 warps in shared memory, the
    // cluster's 8 CTAs through distributed shared memory
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        acc[e] = __dadd_rn(acc[e], __shfl_xor_sync(0xffffffffu, acc[e], 8));
        acc[e] = __dadd_rn(acc[e], __shfl_xor_sync(0xffffffffu, acc[e], 16));
    }
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) < kStatsTPR) {
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp][cc * 8 + e] = acc[e];
    }
    __syncthreads();
    if (threadIdx.x < kStatsCols) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < kStatsWarps; ++w) s = __dadd_rn(s, red[w][threadIdx.x]);
        part[threadIdx.x] = s;
    }
    cluster.sync();
    if (rank == 0 && threadIdx.x < kStatsCols) {
        double s = 0.0;
        for (int q = 0; q < kStatsCluster; ++q)
            s = __dadd_rn(s, *cluster.map_shared_rank(&part[threadIdx.x], q));
        const int64_t col = (int64_t)slab * kStatsCols + threadIdx.x;
        if (col < K) a[col] = __double2float_rn(__ddiv_rn(s, (double)T));
    }
    cluster.sync();   // keep every CTA's shared memory alive until CTA 0 has read it
}

// ===========================================================================
// a2. Search space: s[i,j] = RN32(pow(max(a_j, FLT_MIN), alpha_i)), evaluated in
//     binary64 ([AWQ-note] "Measures": compute a^alpha for each candidate),
//     and its reciprocal rs = RN32(1/s) used to undo the scaling.
// ===========================================================================
__global__ void alpha_scales_kernel(const float *__restrict__ a, int64_t K,
                                    const float *__restrict__ alphas, int n_alpha,
                                    float *__restrict__ s, float *__restrict__ rs) {
    const int64_t total = (int64_t)n_alpha * K;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int ai = (int)(i / K);
        const int64_t j = i - (int64_t)ai * K;
        const float al = alphas[ai];
        if (!(al >= 0.0f && al <= 1.0f)) atomicOr(&g_dev_error, kDevErrBadAlpha);
        const float aj = fmaxf(a[j], FLT_MIN);
        const float sv = __double2float_rn(pow((double)aj, (double)al));
        s[i] = sv;
        if (rs) rs[i] = __frcp_rn(sv);
    }
}

// ===========================================================================
// a3 (group half). For every (alpha, row, group): min/max of w' = RN32(w*s) and
// the quantizer parameters ([QAS-QA] §5, §9).  A block owns one column group
// and 128 / LPR rows; each lane holds 64 consecutive weights of one row as
// binary32 in registers (LPR = group/64 lanes per row) and walks the whole
// alpha grid, reading the group's s values -- staged once per block in shared
// memory, where all lanes of a warp read the same address -- so W is read once
// and s is not re-fetched per row.  Layout of the result:
// params[(alpha * G + group) * N_pad + row]; rows [N, N_pad) get zeros.
// ===========================================================================
constexpr int kGpThreads = 128;
constexpr int kGpCols = 64;              // columns per lane

__device__ __forceinline__ void load_row64(const __half *src, float (&w)[kGpCols]) {
#pragma unroll
    for (int q = 0; q < kGpCols / 8; ++q) {
        const uint4 v = ldg_stream_v4(src + 8 * q);
        const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            w[8 * q + 2 * e] = f.x;
            w[8 * q + 2 * e + 1] = f.y;
        }
    }
}

// min and max of w[k] * s[k] over the lane's 64 columns (s in shared memory),
// in four independent chains so that consecutive min/max operations do not
// wait on one another (min and max are exact, so the grouping is free).
__device__ __forceinline__ void minmax64(const float (&w)[kGpCols], const float *s_sm, float &mn, float &mx) {
    float lo[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
    float hi[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int q = 0; q < kGpCols / 4; ++q) {
        const float4 sv = *reinterpret_cast<const float4 *>(s_sm + 4 * q);
        const float2 p0 = mul2_rn(make_float2(w[4 * q], w[4 * q + 1]), make_float2(sv.x, sv.y));
        const float2 p1 = mul2_rn(make_float2(w[4 * q + 2], w[4 * q + 3]), make_float2(sv.z, sv.w));
        // two three-input operations per four products and per bound
        lo[q & 3] = fmin3(fmin3(lo[q & 3], p0.x, p0.y), p1.x, p1.y);
        hi[q & 3] = fmax3(fmax3(hi[q & 3], p0.x, p0.y), p1.x, p1.y);
    }
    mn = fminf(fmin3(lo[0], lo[1], lo[2]), lo[3]);
    mx = fmaxf(fmax3(hi[0], hi[1], hi[2]), hi[3]);
}

// The same over the channels not held in fp16 (keep: one flag byte per column
// in shared memory); a lane whose columns are all kept returns +inf / -inf.
__device__ __forceinline__ void minmax64_kept(const float (&w)[kGpCols], const float *s_sm, const uint8_t *keep,
                                              float &mn, float &mx) {
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll
    for (int k = 0; k < kGpCols; ++k) {
        const float p = __fmul_rn(w[k], s_sm[k]);
        lo = keep[k] ? lo : fminf(lo, p);
        hi = keep[k] ? hi : fmaxf(hi, p);
    }
    mn = lo;
    mx = hi;
}

template <int LPR>   // lanes per row = group_size / 64
__global__ void __launch_bounds__(kGpThreads, 3)
group_params_kernel(const __half *__restrict__ W, int64_t N, int64_t N_pad, int64_t K, int G,
                    const float *__restrict__ s_tab, int n_alpha, float qmax, int sym,
                    const uint8_t *__restrict__ mask, uint2 *__restrict__ params) {
    __shared__ uint8_t keep_sm[LPR * kGpCols];
    extern __shared__ float s_sm[];                 // [n_alpha][LPR][kGpCols + 4] (+4: the halves sit in other banks)
    constexpr int kRowsPerBlock = kGpThreads / LPR;
    constexpr int kStride = kGpCols + 4;
    const int grp = blockIdx.x % G;
    const int64_t n0 = (int64_t)(blockIdx.x / G) * kRowsPerBlock;
    const int64_t k0 = (int64_t)grp * (kGpCols * LPR);
    for (int i = threadIdx.x; i < n_alpha * LPR * kGpCols; i += kGpThreads) {
        const int ai = i / (LPR * kGpCols), rem = i % (LPR * kGpCols);
        s_sm[(ai * LPR + rem / kGpCols) * kStride + rem % kGpCols] = __ldg(s_tab + (int64_t)ai * K + k0 + rem);
    }
    if (mask)
        for (int i = threadIdx.x; i < LPR * kGpCols; i += kGpThreads) keep_sm[i] = __ldg(mask + k0 + i);
    __syncthreads();
    const int half = threadIdx.x % LPR;
    const int64_t n = n0 + threadIdx.x / LPR;
    const bool active = n < N;
    float w[kGpCols];
    if (active) {
        load_row64(W + n * K + k0 + half * kGpCols, w);
    } else {
#pragma unroll
        for (int e = 0; e < kGpCols; ++e) w[e] = 0.0f;
    }
    // two alphas per iteration: their chains (products, min/max, the divide and
    // reciprocal of the parameters) are independent and interleave
    for (int a0 = 0; a0 < n_alpha; a0 += 2) {
        const int na = n_alpha - a0 < 2 ? 1 : 2;
        float mn[2], mx[2];
#pragma unroll
        for (int d = 0; d < 2; ++d) {
            const int ai = d < na ? a0 + d : a0;
            if (mask)
                minmax64_kept(w, s_sm + (ai * LPR + half) * kStride, keep_sm + half * kGpCols, mn[d], mx[d]);
            else
                minmax64(w, s_sm + (ai * LPR + half) * kStride, mn[d], mx[d]);
        }
#pragma unroll
        for (int d = 0; d < 2; ++d) {
            if (LPR == 2) {
                mn[d] = fminf(mn[d], __shfl_xor_sync(0xffffffffu, mn[d], 1));
                mx[d] = fmaxf(mx[d], __shfl_xor_sync(0xffffffffu, mx[d], 1));
            }
            if (mn[d] > mx[d]) { mn[d] = 0.0f; mx[d] = 0.0f; }   // every channel of the group kept in fp16
        }
        if (LPR == 2) {
            // the row's two lanes share the work: lane `half` derives and stores alpha a0 + half
            const float lo_ = half ? mn[1] : mn[0], hi_ = half ? mx[1] : mx[0];
            const uint2 v = active ? pack_qparams(make_qparams(lo_, hi_, qmax, sym != 0)) : make_uint2(0, 0);
            if (half < na && n < N_pad) params[((int64_t)(a0 + half) * G + grp) * N_pad + n] = v;
        } else {
            uint2 v[2];
#pragma unroll
            for (int d = 0; d < 2; ++d)
                v[d] = active ? pack_qparams(make_qparams(mn[d], mx[d], qmax, sym != 0)) : make_uint2(0, 0);
            if (n < N_pad) {
#pragma unroll
                for (int d = 0; d < 2; ++d)
                    if (d < na) params[((int64_t)(a0 + d) * G + grp) * N_pad + n] = v[d];
            }
        }
    }
}

// ===========================================================================
// a3/a4 standalone: W_hat = RN16(RN32(RN32((q - z) sh) * RN32(1/s))) for one s.
// ===========================================================================
template <int TPG>
__global__ void __launch_bounds__(256)
quant_dequant_kernel(const __half *__restrict__ W, int64_t N, int64_t K, int G,
                     const float *__restrict__ s, float qmax, int sym, const uint8_t *__restrict__ mask,
                     __half *__restrict__ W_hat) {
    const int64_t gid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / TPG;
    const int sub = threadIdx.x % TPG;
    const bool active = gid < N * (int64_t)G;
    const int64_t n = active ? gid / G : 0;
    const int grp = active ? (int)(gid - n * G) : 0;
    const int64_t k0 = (int64_t)grp * (TPG * 16) + sub * 16;
    float wv[16], sv[16], wp[16], rs[16];
    {
        uint4 v0 = active ? ldg_stream_v4(W + n * K + k0) : make_uint4(0, 0, 0, 0);
        uint4 v1 = active ? ldg_stream_v4(W + n * K + k0 + 8) : make_uint4(0, 0, 0, 0);
        const __half *h0 = reinterpret_cast<const __half *>(&v0);
        const __half *h1 = reinterpret_cast<const __half *>(&v1);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            sv[e] = active ? __ldg(s + k0 + e) : 1.0f;
            wv[e] = __half2float(e < 8 ? h0[e] : h1[e - 8]);
            wp[e] = __fmul_rn(wv[e], sv[e]);
            rs[e] = __frcp_rn(sv[e]);
        }
    }
    bool kept[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) kept[e] = mask && active && __ldg(mask + k0 + e) != 0;
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        mn = kept[e] ? mn : fminf(mn, wp[e]);
        mx = kept[e] ? mx : fmaxf(mx, wp[e]);
    }
#pragma unroll
    for (int off = 1; off < TPG; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    if (mn > mx) { mn = 0.0f; mx = 0.0f; }              // every channel of the group kept in fp16
    const QParams prm = make_qparams(mn, mx, qmax, sym != 0);
    const QPair qp = make_qpair(prm, qmax);
    if (!active) return;
    __align__(16) __half2 out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        out[e] = prm.clamp
                     ? dequant_unscale_pair<true>(make_float2(wv[2 * e], wv[2 * e + 1]),
                                                  make_float2(sv[2 * e], sv[2 * e + 1]),
                                                  make_float2(rs[2 * e], rs[2 * e + 1]), qp)
                     : dequant_unscale_pair<false>(make_float2(wv[2 * e], wv[2 * e + 1]),
                                                   make_float2(sv[2 * e], sv[2 * e + 1]),
                                                   make_float2(rs[2 * e], rs[2 * e + 1]), qp);
    if (mask) {                                      // channels kept in fp16 pass through
        __half *o = reinterpret_cast<__half *>(out);
#pragma unroll
        for (int e = 0; e < 16; ++e)
            if (kept[e]) o[e] = __float2half_rn(wv[e]);
    }
    *reinterpret_cast<uint4 *>(W_hat + n * K + k0) = *reinterpret_cast<const uint4 *>(&out[0]);
    *reinterpret_cast<uint4 *>(W_hat + n * K + k0 + 8) = *reinterpret_cast<const uint4 *>(&out[4]);
}

// ===========================================================================
// Quantizer variants and baselines ([AWQ-note] "Measures": RTN, a fixed scale
// of 2 on the salient channels, and keeping 1% of the channels in FP16,
// chosen by activation or by weight magnitude).
// ===========================================================================

// A caller's scale table s[i][k] (scales given instead of a^alpha): copied
// into the workspace with rs = RN32(1/s); a scale that is not a positive
// finite number raises the bad-scale flag (the search would be meaningless).
__global__ void scale_table_kernel(const float *__restrict__ s_in, int64_t total, float *__restrict__ s_tab,
                                   float *__restrict__ rs_tab) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = s_in[i];
        if (!(v > 0.0f && v <= FLT_MAX)) atomicOr(&g_dev_error, kDevErrBadScale);
        s_tab[i] = v;
        rs_tab[i] = __frcp_rn(v);
    }
}

// Xm = X with the columns of the channels kept in fp16 set to +0: their
// error is zero, so they must not reach the loss (the search contracts
// W_hat - W against Xm).  8 columns per thread, 16-byte accesses.
__global__ void mask_columns_kernel(const __half *__restrict__ X, int64_t T, int64_t K, int64_t ldx,
                                    const uint8_t *__restrict__ mask, __half *__restrict__ Xm) {
    const int64_t per_row = K / 8, total = T * per_row;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_row, c = (i - t * per_row) * 8;
        uint4 v = ldg_stream_v4(X + t * ldx + c);
        const uint2 m = *reinterpret_cast<const uint2 *>(mask + c);
        uint16_t *h = reinterpret_cast<uint16_t *>(&v);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if ((e < 4 ? (m.x >> (8 * e)) : (m.y >> (8 * (e - 4)))) & 0xFFu) h[e] = 0;
        *reinterpret_cast<uint4 *>(Xm + t * K + c) = v;
    }
}

// s[k] = factor for the channels in the mask, 1 elsewhere: the variant that
// scales only the salient channels by a fixed factor ([AWQ-note] "Measures":
// scaling them by 2 instead of keeping them in FP16).
__global__ void salient_scales_kernel(const uint8_t *__restrict__ mask, int64_t K, float factor,
                                      float *__restrict__ s) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < K; i += (int64_t)gridDim.x * blockDim.x)
        s[i] = mask[i] ? factor : 1.0f;
}

// mask[j] = 1 for the k channels of largest stat[j] (ties: lower index first;
// NaN ranks below every number), by counting, for each j, the channels that
// come before it.  A block stages a tile of the statistic in shared memory;
// K^2 comparisons, microseconds for the layers here.
constexpr int kTopkThreads = 256;
__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float *__restrict__ stat, int64_t K, int64_t k, uint8_t *__restrict__ mask) {
    __shared__ float tile[kTopkThreads];
    const int64_t j = blockIdx.x * (int64_t)kTopkThreads + threadIdx.x;
    const float vj = j < K ? stat[j] : 0.0f;
    const bool nj = isnan(vj);
    int64_t before = 0;
    for (int64_t i0 = 0; i0 < K; i0 += kTopkThreads) {
        __syncthreads();
        tile[threadIdx.x] = i0 + threadIdx.x < K ? stat[i0 + threadIdx.x] : 0.0f;
        __syncthreads();
        const int lim = (int)(K - i0 < kTopkThreads ? K - i0 : kTopkThreads);
        for (int q = 0; q < lim; ++q) {
            const int64_t i = i0 + q;
            const float vi = tile[q];
            const bool ni = isnan(vi);
            bool b;
            if (ni || nj) b = (!ni && nj) || (ni && nj && i < j);
            else b = vi > vj || (vi == vj && i < j);
            before += (i != j && b) ? 1 : 0;
        }
    }
    if (j < K) mask[j] = before < k ? 1 : 0;
}

// ===========================================================================
// a4-a6 on a CTA pair.  Two CTAs of a cluster share one tcgen05 cta_group::2
// MMA of M = 256 (each CTA owns 128 W rows of the unit) by N = 256 tokens
// (each CTA holds 128 of them), two accumulators side by side: a work unit is
// 256 W rows x 512 tokens for one alpha.  Per CTA and 64-column k-step:
//   * the X warp TMA-loads this CTA's two 128-token halves (32 KiB) and counts
//     their bytes on the leader's full barrier;
//   * the W warp TMA-loads the CTA's W tile (128 x 64, 128-byte swizzle), its
//     1 KiB of group parameters and 64 s and 1/s values into a 4-deep ring, so
//     the producer reads everything from shared memory;
//   * 8 producer warps build Delta W = W_hat - W in the A tile and arrive on
//     their own CTA's A barrier; in the peer one thread forwards a single
//     cluster-scope arrive per stage to the leader (9 arrivals per stage);
//   * the leader's MMA thread issues the pair MMAs and releases both CTAs'
//     stages with one multicast commit; the epilogue of each CTA drains its
//     own 128 TMEM lanes and tells the leader (8 arrivals per unit).
// Halving the X tile per SM (against one CTA doing M = 128) is what frees the
// shared memory for the W ring.
// ===========================================================================
namespace srch2 {
constexpr int BM = 128;                 // W rows per CTA
constexpr int PM = 2 * BM;              // W rows per unit (MMA M)
constexpr int BN = 256;                 // tokens per MMA (MMA N, 128 per CTA)
constexpr int HN = BN / 2;
constexpr int NJ = 2;                   // accumulators per unit
constexpr int BT = BN * NJ;             // tokens per unit
constexpr int BK = 64;                  // K per stage (one 128-byte swizzled row)
constexpr int XS = 3, AS = 3, WS = 4;   // ring depths
constexpr int X_J_BYTES = HN * BK * 2;               // 16 KiB
constexpr int X_STAGE_BYTES = NJ * X_J_BYTES;        // 32 KiB per CTA
constexpr int A_STAGE_BYTES = BM * BK * 2;           // 16 KiB
constexpr int W_TILE_BYTES = BM * BK * 2;            // 16 KiB
constexpr int PRM_BYTES = BM * 8;                    // 1 KiB
constexpr int SV_BYTES = BK * 4;                     // 256 B
constexpr int W_TX_BYTES = W_TILE_BYTES + PRM_BYTES + 2 * SV_BYTES;
constexpr int NUM_EPI_WARPS = 4;
constexpr int XTMA_WARP = 4;
constexpr int MMA_WARP = 5;
constexpr int WTMA_WARP = 6;
constexpr int PROD_WARP0 = 8;
constexpr int NUM_PROD_WARPS = 8;
constexpr int NUM_THREADS = (PROD_WARP0 + NUM_PROD_WARPS) * 32;   // 512
constexpr int TMEM_COLS = 512;
constexpr uint32_t IDESC = mma_idesc_f16_f32(PM, BN);
constexpr uint16_t PAIR_MASK = 0x3;

struct Smem {
    uint8_t x[XS][X_STAGE_BYTES];       // every tile 1024-byte aligned
    uint8_t a[AS][A_STAGE_BYTES];
    uint8_t w[WS][W_TILE_BYTES];
    uint2 prm[WS][BM];
    float sv[WS][BK];
    float rsv[WS][BK];
    uint64_t x_full[XS], x_empty[XS];
    uint64_t a_full[AS], a_empty[AS];
    uint64_t w_full[WS], w_empty[WS];
    uint64_t acc_full[NJ], acc_empty[NJ], drain;
    uint32_t tmem_base;
    int abort_flag;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;

struct Args {
    const uint2 *params;        // [n_alpha][G][N_pad]
    const float *s_tab;         // [n_alpha][K]
    const float *rs_tab;        // [n_alpha][K]
    float *partial;             // [n_alpha][n_tb][N]
    int64_t N, K, T, N_pad;
    int n_alpha, G, group;
    int n_tb, n_kb;
    int64_t n_units;
    float qmax;
    uint64_t timeout_ns;
};

struct UnitIdx { int nb, tb, alpha; };
__device__ __forceinline__ UnitIdx unit_index(int64_t u, const Args &A) {
    UnitIdx r;
    const int64_t tile = u / A.n_alpha;
    r.alpha = (int)(u - tile * A.n_alpha);
    r.nb = (int)(tile / A.n_tb);
    r.tb = (int)(tile - (int64_t)r.nb * A.n_tb);
    return r;
}

// Delta W = W_hat - W (fp16) for this thread's slice of a stage: 4 rows x 8
// consecutive weights, all 16 pairs in one unrolled block so their dependency
// chains interleave.  kClamp selects the code-clamping variant; the warp takes
// it only when one of its rows has a group that needs it (about 0.1% of groups
// on LLM-like weights, so ~2% of stages).
template <bool kClamp>
__device__ __forceinline__ void compute_stage(const uint4 (&w)[4], const QParams (&qp)[4], const float4 (&sv)[2],
                                              const float4 (&rv)[2], float qmax, uint4 (&out)[4]) {
    const float2 s4[4] = {make_float2(sv[0].x, sv[0].y), make_float2(sv[0].z, sv[0].w),
                          make_float2(sv[1].x, sv[1].y), make_float2(sv[1].z, sv[1].w)};
    const float2 r4[4] = {make_float2(rv[0].x, rv[0].y), make_float2(rv[0].z, rv[0].w),
                          make_float2(rv[1].x, rv[1].y), make_float2(rv[1].z, rv[1].w)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const QPair q = make_qpair(qp[i], qmax);
        const __half2 *wh = reinterpret_cast<const __half2 *>(&w[i]);
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const __half2 d = __hsub2(dequant_unscale_pair<kClamp>(__half22float2(wh[p]), s4[p], r4[p], q), wh[p]);
            o[p] = *reinterpret_cast<const uint32_t *>(&d);
        }
        out[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
search_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const Args A) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int64_t pair = blockIdx.x >> 1;
    const int64_t npairs = gridDim.x >> 1;
    volatile int *abort_flag = &S.abort_flag;

    if (threadIdx.x == 0) {
        for (int i = 0; i < XS; ++i) { mbar_init(&S.x_full[i], 1); mbar_init(&S.x_empty[i], 1); }
        // leader: its 8 producer warps + one forwarded arrival from the peer; peer: its 8 producer warps
        for (int i = 0; i < AS; ++i) {
            mbar_init(&S.a_full[i], leader ? NUM_PROD_WARPS + 1 : NUM_PROD_WARPS);
            mbar_init(&S.a_empty[i], 1);
        }
        for (int i = 0; i < WS; ++i) { mbar_init(&S.w_full[i], 1); mbar_init(&S.w_empty[i], NUM_PROD_WARPS); }
        for (int j = 0; j < NJ; ++j) {
            mbar_init(&S.acc_full[j], 1);
            mbar_init(&S.acc_empty[j], 2 * NUM_EPI_WARPS);
        }
        mbar_init(&S.drain, 1);
        S.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == XTMA_WARP) {
        tmem_alloc_pair(&S.tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
        tc_fence_before();
    }
    __syncthreads();
    cluster_sync_all();      // both CTAs' barriers exist before anyone signals across the pair
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    bool aborted = false;

    if (warp == XTMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tmap_x);
            int xs = 0;
            uint32_t xph = 0;
            for (int64_t u = pair; u < A.n_units && !aborted; u += npairs) {
                const UnitIdx ui = unit_index(u, A);
                const int t0 = ui.tb * BT + (int)rank * HN;
                for (int kb = 0; kb < A.n_kb; ++kb) {
                    if (!mbar_wait_bounded(&S.x_empty[xs], xph ^ 1u, abort_flag, A.timeout_ns)) { aborted = true; break; }
                    if (leader) mbar_arrive_expect_tx(&S.x_full[xs], 2 * X_STAGE_BYTES);
                    const uint32_t full_l = mapa_shared(smem_u32(&S.x_full[xs]), 0);
#pragma unroll
                    for (int j = 0; j < NJ; ++j)
                        tma_load_2d_pair(&S.x[xs][j * X_J_BYTES], &tmap_x, kb * BK, t0 + j * BN, full_l);
                    if (++xs == XS) { xs = 0; xph ^= 1u; }
                }
            }
        }
    } else if (warp == WTMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tmap_w);
            int ws = 0;
            uint32_t wph = 0;
            for (int64_t u = pair; u < A.n_units && !aborted; u += npairs) {
                const UnitIdx ui = unit_index(u, A);
                const int n0 = ui.nb * PM + (int)rank * BM;
                for (int kb = 0; kb < A.n_kb; ++kb) {
                    if (!mbar_wait_bounded(&S.w_empty[ws], wph ^ 1u, abort_flag, A.timeout_ns)) { aborted = true; break; }
                    mbar_arrive_expect_tx(&S.w_full[ws], W_TX_BYTES);
                    tma_load_2d(&S.w[ws][0], &tmap_w, kb * BK, n0, &S.w_full[ws]);
                    const int grp = (int)(((int64_t)kb * BK) / A.group);
                    bulk_load(&S.prm[ws][0], A.params + ((int64_t)ui.alpha * A.G + grp) * A.N_pad + n0, PRM_BYTES,
                              &S.w_full[ws]);
                    bulk_load(&S.sv[ws][0], A.s_tab + (int64_t)ui.alpha * A.K + (int64_t)kb * BK, SV_BYTES,
                              &S.w_full[ws]);
                    bulk_load(&S.rsv[ws][0], A.rs_tab + (int64_t)ui.alpha * A.K + (int64_t)kb * BK, SV_BYTES,
                              &S.w_full[ws]);
                    if (++ws == WS) { ws = 0; wph ^= 1u; }
                }
            }
        }
    } else if (warp == MMA_WARP && !leader) {
        // Peer: forward "my half of A stage `as` is written" to the leader with a
        // single cluster-scope arrive per stage (the producers arrive locally,
        // with cheap CTA-scope release; release is cumulative, so this arrive
        // also orders their writes for the leader's MMA).
        if (lane == 0) {
            int as = 0;
            uint32_t aph = 0;
            for (int64_t u = pair; u < A.n_units && !aborted; u += npairs) {
                for (int kb = 0; kb < A.n_kb; ++kb) {
                    if (!mbar_wait_bounded(&S.a_full[as], aph, abort_flag, A.timeout_ns)) { aborted = true; break; }
                    mbar_arrive_cluster(mapa_shared(smem_u32(&S.a_full[as]), 0));
                    if (++as == AS) { as = 0; aph ^= 1u; }
                }
            }
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) {
            int xs = 0, as = 0;
            uint32_t xph = 0, aph = 0, accph = 0;
            // The two accumulators are handed over separately: accumulator j of a
            // unit is committed right after its last MMAs and reused by the next
            // unit as soon as the epilogue has drained it, so one accumulator's
            // drain overlaps the other's MMAs.
            for (int64_t u = pair; u < A.n_units && !aborted; u += npairs) {
                for (int kb = 0; kb < A.n_kb && !aborted; ++kb) {
                    if (!mbar_wait_bounded(&S.a_full[as], aph, abort_flag, A.timeout_ns) ||
                        !mbar_wait_bounded(&S.x_full[xs], xph, abort_flag, A.timeout_ns)) { aborted = true; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(&S.a[as][0]);
                    const uint32_t x_base = smem_u32(&S.x[xs][0]);
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        if (kb == 0) {
                            if (!mbar_wait_bounded(&S.acc_empty[j], accph ^ 1u, abort_flag, A.timeout_ns)) {
                                aborted = true;
                                break;
                            }
                            tc_fence_after();
                        }
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t adesc = sw128_kmajor_desc(a_base + kk * 32);
                            const uint64_t bdesc = sw128_kmajor_desc(x_base + j * X_J_BYTES + kk * 32);
                            mma_f16_ss_pair(tmem + j * BN, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
                        }
                        if (kb + 1 == A.n_kb) mma_commit_pair_mc(&S.acc_full[j], PAIR_MASK);
                    }
                    if (aborted) break;
                    mma_commit_pair_mc(&S.x_empty[xs], PAIR_MASK);
                    mma_commit_pair_mc(&S.a_empty[as], PAIR_MASK);
                    if (++xs == XS) { xs = 0; xph ^= 1u; }
                    if (++as == AS) { as = 0; aph ^= 1u; }
                }
                accph ^= 1u;
            }
            mma_commit_pair(&S.drain);                  // every pair MMA of this thread done before teardown
            mbar_wait_bounded(&S.drain, 0, abort_flag, A.timeout_ns);
        }
    } else if (warp < NUM_EPI_WARPS) {
        uint32_t accph = 0;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        for (int64_t u = pair; u < A.n_units && !aborted; u += npairs) {
            const UnitIdx ui = unit_index(u, A);
            float2 sum2 = make_float2(0.0f, 0.0f);
#pragma unroll 1
            for (int j = 0; j < NJ; ++j) {
                if (!mbar_wait_warp(&S.acc_full[j], accph, abort_flag, A.timeout_ns, 256)) { aborted = true; break; }
                tc_fence_after();
#pragma unroll 1
                for (int c = j * BN; c < (j + 1) * BN; c += 64) {
                    float v[64];
                    tmem_ld_32x32b_x64_sync(tmem + lane_base + c, v);
#pragma unroll
                    for (int i = 0; i < 64; i += 2) {
                        const float2 e = make_float2(v[i], v[i + 1]);
                        sum2 = fma2_rn(e, e, sum2);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader) mbar_arrive(&S.acc_empty[j]);
                    else mbar_arrive_cluster(mapa_shared(smem_u32(&S.acc_empty[j]), 0));
                }
            }
            if (aborted) break;
            const float sum = __fadd_rn(sum2.x, sum2.y);
            const int64_t n = (int64_t)ui.nb * PM + rank * BM + warp * 32 + lane;
            if (n < A.N) A.partial[((int64_t)ui.alpha * A.n_tb + ui.tb) * A.N + n] = sum;
            accph ^= 1u;
        }
    } else if (warp >= PROD_WARP0) {
        const int p = threadIdx.x - PROD_WARP0 * 32;   // 0..255
        const int c = p & 7;                            // 16-byte chunk of the 128-byte row
        const int rbase = p >> 3;                       // rows rbase + 32 i
        int ws = 0, as = 0;
        uint32_t wph = 0, aph = 0;
        for (int64_t u = pair; u < A.n_units && !aborted; u += npairs) {
            for (int kb = 0; kb < A.n_kb; ++kb) {
                if (!mbar_wait_warp(&S.w_full[ws], wph, abort_flag, A.timeout_ns)) { aborted = true; break; }
                const uint32_t wb = smem_u32(&S.w[ws][0]);
                uint4 w[4];
                QParams qp[4];
                bool need = false;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    w[i] = lds_v4(wb + sw128_offset(rbase + 32 * i, c));
                    qp[i] = unpack_qparams(lds_v2(smem_u32(&S.prm[ws][rbase + 32 * i])));
                    need |= qp[i].clamp;
                }
                float4 sv[2], rv[2];
                sv[0] = lds_f4(smem_u32(&S.sv[ws][c * 8]));
                sv[1] = lds_f4(smem_u32(&S.sv[ws][c * 8 + 4]));
                rv[0] = lds_f4(smem_u32(&S.rsv[ws][c * 8]));
                rv[1] = lds_f4(smem_u32(&S.rsv[ws][c * 8 + 4]));
                uint4 outv[4];
                if (__any_sync(0xffffffffu, need))
                    compute_stage<true>(w, qp, sv, rv, A.qmax, outv);
                else
                    compute_stage<false>(w, qp, sv, rv, A.qmax, outv);
                // Release the stage only now: an issued shared-memory load is complete
                // once an instruction has consumed its register, and every value read
                // from the stage has been consumed by the arithmetic above.  (An arrive
                // right after the loads could let the next tile's copy overwrite the
                // stage under a load still in flight.)
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.w_empty[ws]);
                if (++ws == WS) { ws = 0; wph ^= 1u; }
                if (!mbar_wait_warp(&S.a_empty[as], aph ^ 1u, abort_flag, A.timeout_ns)) { aborted = true; break; }
                const uint32_t a_base = smem_u32(&S.a[as][0]);
#pragma unroll
                for (int i = 0; i < 4; ++i) st_shared_v4(a_base + sw128_offset(rbase + 32 * i, c), outv[i]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.a_full[as]);      // local; the peer's is forwarded
                if (++as == AS) { as = 0; aph ^= 1u; }
            }
        }
    }

    // On an abort, give copies already in flight time to land before the CTA
    // can leave (bounded: about 200 microseconds).
    if (aborted || *abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();      // neither CTA leaves while its pair may still signal it or read its tiles
    if (warp == XTMA_WARP) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}
}  // namespace srch2

// ===========================================================================
// a6 (reduction). losses[i] = RN32(sum over token blocks and rows of the
// partials, in binary64 and a fixed order, / (R T)), R = N for a whole layer
// or the layer's row count when these N rows are one part of it; optional
// per-row sums.  One block per alpha; thread t takes rows t, t + 1024, ... in
// that order, kLossRows of them at a time so that all their loads of a batch
// of 8 token blocks are in flight together.
// ===========================================================================
constexpr int kLossThreads = 1024;
constexpr int kLossRows = 2;
__global__ void __launch_bounds__(kLossThreads)
loss_reduce_kernel(const float *__restrict__ partial, int64_t N, int64_t T, int n_tb, int64_t norm_rows,
                   float *__restrict__ losses, float *__restrict__ row_losses) {
    const int ai = blockIdx.x;
    const float *p = partial + (int64_t)ai * n_tb * N;
    double acc = 0.0;
    for (int64_t nb = threadIdx.x; nb < N; nb += kLossRows * kLossThreads) {
        float rsum[kLossRows];
        double dsum[kLossRows];
#pragma unroll
        for (int i = 0; i < kLossRows; ++i) { rsum[i] = 0.0f; dsum[i] = 0.0; }
        for (int tb0 = 0; tb0 < n_tb; tb0 += 8) {
            float v[kLossRows][8];
#pragma unroll
            for (int i = 0; i < kLossRows; ++i) {
                const int64_t n = nb + (int64_t)i * kLossThreads;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    v[i][j] = (n < N && tb0 + j < n_tb) ? __ldg(p + (int64_t)(tb0 + j) * N + n) : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < kLossRows; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    rsum[i] = __fadd_rn(rsum[i], v[i][j]);
                    dsum[i] = __dadd_rn(dsum[i], (double)v[i][j]);
                }
        }
#pragma unroll
        for (int i = 0; i < kLossRows; ++i) {
            const int64_t n = nb + (int64_t)i * kLossThreads;
            if (n < N) {
                if (row_losses) row_losses[(int64_t)ai * N + n] = rsum[i];
                acc = __dadd_rn(acc, dsum[i]);
            }
        }
    }
    __shared__ double red[kLossThreads];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int off = kLossThreads / 2; off > 0; off >>= 1) {
        if ((int)threadIdx.x < off) red[threadIdx.x] = __dadd_rn(red[threadIdx.x], red[threadIdx.x + off]);
        __syncthreads();
    }
    if (threadIdx.x == 0) losses[ai] = __double2float_rn(red[0] / ((double)norm_rows * (double)T));
}

// ===========================================================================
// a7. Argmin over the grid (first index, NaN = +inf) and s at the best alpha.
// Every block re-derives the argmin from the n_alpha losses (no host round trip).
// ===========================================================================
__device__ __forceinline__ int argmin_losses(const float *losses, int n) {
    int best = 0;
    float bv = INFINITY;
    bool have = false;
    for (int i = 0; i < n; ++i) {
        float v = losses[i];
        if (isnan(v)) v = INFINITY;
        if (!have || v < bv) { bv = v; best = i; have = true; }
    }
    return best;
}

__global__ void best_scale_kernel(const float *__restrict__ a, int64_t K,
                                  const float *__restrict__ alphas,
                                  const float *__restrict__ losses, int n_alpha,
                                  int32_t *__restrict__ best_idx, float *__restrict__ s_best) {
    __shared__ int sb;
    if (threadIdx.x == 0) {
        sb = argmin_losses(losses, n_alpha);
        if (blockIdx.x == 0) *best_idx = sb;
    }
    __syncthreads();
    const float al = alphas[sb];
    if (!(al >= 0.0f && al <= 1.0f) && threadIdx.x == 0) atomicOr(&g_dev_error, kDevErrBadAlpha);
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < K;
         j += (int64_t)gridDim.x * blockDim.x) {
        const float aj = fmaxf(a[j], FLT_MIN);
        s_best[j] = __double2float_rn(pow((double)aj, (double)al));
    }
}

// ===========================================================================
// a8. Pack: per (row, group) recompute w' = RN32(w s_best), the group's
// parameters and every code; store codes LSB-first, the fp16 scale and zero
// ([AWQ-note] "Measures": keep the quantized weights and their metadata).
// A warp takes items of 4 rows x 256 columns; lane l holds columns 8l..8l+7
// of each row, so every load instruction of the warp reads 512 contiguous
// bytes of one row and every code store writes the row's words contiguously.
// A group of g columns is GL = g/8 neighbouring lanes.  Its min and max go
// through a reduce-scatter over those lanes (lane i of a group ends with row
// i mod 4's values), each lane computes the parameters of that one row, and
// the lanes of the group read them back by shuffles.  HBM-bound: W is read
// once, codes, scales and zeros are written once.
// ===========================================================================
constexpr int kPkThreads = 256;
constexpr int kPkRows = 4;               // rows per warp item (4: fewer registers, more warps resident)
constexpr int kPkCols = 256;             // columns per warp item (8 per lane)

// min over the GL lanes of this lane's group of v[i], for i = this lane's row
// (lane index within the group mod kPkRows); max likewise.  kPkRows <= 8 = the
// smallest group's lane count.
template <int GL>
__device__ __forceinline__ void group_reduce_scatter(float (&lo)[kPkRows], float (&hi)[kPkRows], float &mn, float &mx) {
    const int gl = threadIdx.x & (GL - 1);
#pragma unroll
    for (int half = kPkRows / 2; half >= 1; half >>= 1) {
        const bool upper = (gl & half) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float slo = upper ? lo[i] : lo[i + half], shi = upper ? hi[i] : hi[i + half];
            const float klo = upper ? lo[i + half] : lo[i], khi = upper ? hi[i + half] : hi[i];
            lo[i] = fminf(klo, __shfl_xor_sync(0xffffffffu, slo, half));
            hi[i] = fmaxf(khi, __shfl_xor_sync(0xffffffffu, shi, half));
        }
    }
    mn = lo[0];
    mx = hi[0];
#pragma unroll
    for (int o = kPkRows; o < GL; o <<= 1) {              // the group's remaining lanes hold the same rows
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
}

template <int GL>   // lanes per group = group_size / 8
__global__ void __launch_bounds__(kPkThreads)
pack_kernel(const __half *__restrict__ W, int64_t N, int64_t K, int G, int bits, int sym,
            const float *__restrict__ s_best, uint32_t *__restrict__ codes,
            __half *__restrict__ scales, __half *__restrict__ zeros) {
    const int lane = threadIdx.x & 31;
    const int gl = lane & (GL - 1);
    const int gbase = lane & ~(GL - 1);
    const float qmax = (float)((1 << bits) - 1);
    const int64_t n_ct = (K + kPkCols - 1) / kPkCols;
    const int64_t n_items = (N + kPkRows - 1) / kPkRows * n_ct;
    const int64_t wid = ((int64_t)blockIdx.x * kPkThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kPkThreads) >> 5;
    for (int64_t item = wid; item < n_items; item += n_warps) {
        const int64_t rb = item / n_ct, ct = item - rb * n_ct;
        const int64_t n0 = rb * kPkRows;
        const int64_t col = ct * kPkCols + lane * 8;
        const bool colok = col < K;           // K is a multiple of the group: whole groups are in or out
        uint4 raw[kPkRows];
#pragma unroll
        for (int r = 0; r < kPkRows; ++r)
            raw[r] = (colok && n0 + r < N) ? ldg_stream_v4(W + (n0 + r) * K + col) : make_uint4(0u, 0u, 0u, 0u);
        float sv[8];
        if (colok) {
            const float4 s0 = __ldg(reinterpret_cast<const float4 *>(s_best + col));
            const float4 s1 = __ldg(reinterpret_cast<const float4 *>(s_best + col + 4));
            sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
            sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) sv[e] = 1.0f;
        }
        float wp[kPkRows][8];                  // w' = RN32(w s)
        float lo[kPkRows], hi[kPkRows];
#pragma unroll
        for (int r = 0; r < kPkRows; ++r) {
            const __half2 *h = reinterpret_cast<const __half2 *>(&raw[r]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 p = mul2_rn(__half22float2(h[e]), make_float2(sv[2 * e], sv[2 * e + 1]));
                wp[r][2 * e] = p.x;
                wp[r][2 * e + 1] = p.y;
            }
            lo[r] = fminf(fmin3(fmin3(wp[r][0], wp[r][1], wp[r][2]), fmin3(wp[r][3], wp[r][4], wp[r][5]), wp[r][6]), wp[r][7]);
            hi[r] = fmaxf(fmax3(fmax3(wp[r][0], wp[r][1], wp[r][2]), fmax3(wp[r][3], wp[r][4], wp[r][5]), wp[r][6]), wp[r][7]);
        }
        float mn, mx;
        group_reduce_scatter<GL>(lo, hi, mn, mx);
        // this lane's row of its group: gl mod kPkRows
        const QParams mine = make_qparams(mn, mx, qmax, sym != 0);
        const uint2 mine_p = pack_qparams(mine);
        const int64_t grp = col / (GL * 8);
        // Codes packed by integer multiply-adds: with v_e = RN32(w'_e r + kMagic)
        // (clamped when the group needs it), q_e = bits(v_e) - base, base =
        // bits(kMagic) - z, and the word sum_e q_e B^e (B = 16 or 4) equals
        // sum_e bits(v_e) B^e - base sum_e B^e modulo 2^32 -- exact, since the
        // word itself fits in 32 bits.
        const uint32_t B = bits == 2 ? 4u : 16u;
        const uint32_t geom = bits == 2 ? 0x5555u : 0x11111111u;      // sum_{e<8} B^e
#pragma unroll
        for (int r = 0; r < kPkRows; ++r) {
            const int src = gbase + r;
            const uint2 pv = make_uint2(__shfl_sync(0xffffffffu, mine_p.x, src), __shfl_sync(0xffffffffu, mine_p.y, src));
            const QParams p = unpack_qparams(pv);
            const int64_t n = n0 + r;
            const uint32_t base = (uint32_t)(__float_as_int(kMagic) - (int)p.z);
            uint32_t acc = 0u, mult = 1u;
            if (__any_sync(0xffffffffu, p.clamp)) {        // some group of this row needs the code clamp
                const float vlo = __fsub_rn(kMagic, p.z), vhi = __fadd_rn(kMagic, __fsub_rn(qmax, p.z));
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float v = fminf(fmaxf(__fmaf_rn(wp[r][e], p.r, kMagic), vlo), vhi);
                    acc += (uint32_t)__float_as_uint(v) * mult;
                    mult *= B;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    acc += (uint32_t)__float_as_uint(__fmaf_rn(wp[r][e], p.r, kMagic)) * mult;
                    mult *= B;
                }
            }
            uint32_t v = acc - base * geom;
            if (bits == 2) {
                v |= __shfl_down_sync(0xffffffffu, v, 1) << 16;      // 16 codes per word: lane pairs
                if (colok && n < N && (lane & 1) == 0) codes[n * (K / 16) + col / 16] = v;
            } else {
                if (colok && n < N) codes[n * (K / 8) + col / 8] = v;
            }
        }
        const int64_t n = n0 + gl;
        if (colok && gl < kPkRows && n < N) {
            scales[n * G + grp] = __float2half_rn(mine.sh);
            zeros[n * G + grp] = __float2half_rn(mine.z);
        }
    }
}

// ===========================================================================
// Consumer of the packed format: the quantized linear layer Y = X W_hat^T for
// a few tokens (decode), read straight from codes, fp16 scales and zeros
// ([AWQ-note] "Tiny Chat": dequantize inside the kernel, never writing fp16
// weights to DRAM).  Definition (fp32 accumulation, order unspecified):
//   Y[t, n] = sum_k x'[t, k] (q[n, k] - z[n, G]) sh[n, G],
//   x'[t, k] = RN32(x[t, k] RN32(1 / s_k))      (1/s folded into the input)
// The work is HBM-bound on the codes (K/2 bytes per row at 4 bits), so the
// kernel is SIMT: codes stream through a TMA ring in shared memory, (q - z) is
// dequantized exactly by byte permutes, and the products are packed fp32
// multiply-adds.
// ===========================================================================
namespace qlv {
constexpr int ROWS = 64;                 // W rows per row block
constexpr int RGROUPS = 8;               // row groups of RPW rows
constexpr int RPW = ROWS / RGROUPS;
constexpr int CWARPS = 2 * RGROUPS;      // consumer warps: a row group x a column half
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int MAX_STAGES = 4;
constexpr int TOKENS = 4;                // most tokens per pass (activations stay in registers)
constexpr int WORDS = 128;               // code words per row per stage (512 B)
constexpr int CODE_BYTES = ROWS * WORDS * 4;                 // 32 KiB
constexpr int MAX_STAGE_COLS = WORDS * 16;                   // columns per stage at 2 bits
constexpr int SLOT_FLOATS = RGROUPS * 32;                    // one partial-sum slot (a row block segment)
constexpr int PAIR_FLOATS = RGROUPS * 2 * 32;                // column-half exchange, 2 slots per row group
constexpr int SMEM_LIMIT = 226 * 1024;         // dynamic shared memory per block (static use stays below 1 KiB)
// One ring stage: codes [ROWS][WORDS] (TMA tile), x' [TT][SC] floats, then
// the fp16 scales and zeros of the stage's gps groups, [2][ROWS][gps].
__host__ __device__ constexpr int stage_bytes(int sc, int tt, int gps) {
    return (CODE_BYTES + tt * sc * 4 + 4 * ROWS * gps + 127) / 128 * 128;
}
__host__ __device__ constexpr int fixed_smem() {
    return PAIR_FLOATS * 4 + (2 * MAX_STAGES + 4 * RGROUPS) * 8 + 128;
}
inline int ring_stages(int sc, int tt, int gps) {
    const int n = (SMEM_LIMIT - fixed_smem()) / stage_bytes(sc, tt, gps);
    return n < MAX_STAGES ? n : MAX_STAGES;
}

struct Args {
    const float *xs;          // x' of this pass's tokens, stage-permuted rows of Kp floats
    int64_t Kp;
    const __half *scales, *zeros;
    int64_t N, K;
    int G, group, T;          // T: tokens of this pass (<= TT)
    int gps;                  // groups per stage
    int n_stages;             // ring depth
    int sz_mode;              // scale/zero copies: 16 = 16-byte, 4 = 4-byte, 2 = plain loads
    int64_t n_steps, units;   // stages per row block; row blocks x n_steps
    float *Y;                 // this pass's output rows, [T][N]
    float *part;              // partial sums of split row blocks, slot rb + b (see the kernel)
    unsigned *cnt;            // [row blocks][RGROUPS] arrival counters, zero between launches
    uint64_t timeout_ns;
};

// The block whose unit range [units*b/grid, units*(b+1)/grid) holds unit u.
__device__ __forceinline__ int64_t block_of(int64_t u, int64_t units, int64_t grid) {
    return ((u + 1) * grid - 1) / units;
}
}  // namespace qlv

// x'[t, k] = RN32(x[t, k] RN32(1 / s_k)) for t < T_pad, stored in the order the
// decode kernel reads a stage of SC = 128 CPW columns: the stage's columns
// split into two halves, each lane owning 2 consecutive code words (2 CPW
// columns) of a half; the 4-column chunk q of word i of lane l in half h sits
// at float4 slot ((2h + i) CPW/4 + q) * 32 + l, so a warp's 16-byte reads of
// one chunk cover 512 contiguous bytes.  Rows t >= T and columns k >= K are
// zero.  Also clears the decode kernel's arrival counters.
__global__ void qlinear_prep_kernel(const __half *__restrict__ X, int64_t T, int64_t T_pad, int64_t K,
                                    int64_t Kp, int64_t ldx, int CPW, const float *__restrict__ s,
                                    float *__restrict__ xs, unsigned *__restrict__ cnt, int64_t n_cnt) {
    const int SC = qlv::WORDS * CPW;
    const int64_t chunks = Kp / 4, total = T_pad * chunks;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    for (int64_t i = i0; i < n_cnt; i += stride) cnt[i] = 0u;
    for (int64_t i = i0; i < total; i += stride) {
        const int64_t t = i / chunks, d = i - t * chunks;
        const int64_t j = d / (SC / 4);
        const int slot = (int)(d - j * (SC / 4));
        const int l = slot % 32, rest = slot / 32;
        const int q = rest % (CPW / 4), wi = (rest / (CPW / 4)) % 2, h = rest / (CPW / 2);
        const int64_t c0 = j * SC + h * (SC / 2) + l * 2 * CPW + wi * CPW + 4 * q;
        float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (t < T && c0 < K) {
            const uint2 hx = *reinterpret_cast<const uint2 *>(X + t * ldx + c0);
            const float4 sv = *reinterpret_cast<const float4 *>(s + c0);
            const float2 x01 = __half22float2(*reinterpret_cast<const __half2 *>(&hx.x));
            const float2 x23 = __half22float2(*reinterpret_cast<const __half2 *>(&hx.y));
            v = make_float4(__fmul_rn(x01.x, __frcp_rn(sv.x)), __fmul_rn(x01.y, __frcp_rn(sv.y)),
                            __fmul_rn(x23.x, __frcp_rn(sv.z)), __fmul_rn(x23.y, __frcp_rn(sv.w)));
        }
        reinterpret_cast<float4 *>(xs)[i] = v;
    }
}

// (q - z) of the 32/CB codes in one 32-bit word as exact binary32 values: each
// code c becomes the float 2^23 + c by placing its byte under the exponent bits
// of 2^23 (one byte permute), and one packed addition of
// noff = (-(2^23 + z), -(2^23 + z)) leaves q - z.
template <int CB>
__device__ __forceinline__ void dequant_word(uint32_t w, float2 noff, float *d) {
    if (CB == 4) {
        const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;   // codes 2b / 2b+1 in byte b
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float2 f = make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7440u | b)),
                                         __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7440u | b)));
            const float2 r = __fadd2_rn(f, noff);
            d[2 * b] = r.x;
            d[2 * b + 1] = r.y;
        }
    } else {
        uint32_t m[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) m[j] = (w >> (2 * j)) & 0x03030303u;     // code 4b + j in byte b of m[j]
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                const float2 f = make_float2(__uint_as_float(__byte_perm(m[j], 0x4B000000u, 0x7440u | b)),
                                             __uint_as_float(__byte_perm(m[j + 1], 0x4B000000u, 0x7440u | b)));
                const float2 r = __fadd2_rn(f, noff);
                d[4 * b + j] = r.x;
                d[4 * b + j + 1] = r.y;
            }
    }
}

// Reduce V values spread over the 32 lanes of a warp so that lane l ends with
// the warp-wide sum of value (l % V) -- a reduce-scatter butterfly.
template <int V>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[V]) {
#pragma unroll
    for (int width = V; width > 1; width >>= 1) {
        const int half = width >> 1;
        const bool upper = (threadIdx.x & half) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
    }
    float x = v[0];
#pragma unroll
    for (int off = V; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// Persistent decode kernel, one block per SM.  The work is a list of units
// (row block of 64 W rows, stage of 1024 columns at 4 bits / 2048 at 2 bits),
// row block major; block b takes the contiguous range
// [units*b/grid, units*(b+1)/grid), so every SM streams the same number of
// code bytes.  Warp 16 feeds a shared-memory ring (up to 4 stages): lane 0
// issues the unit's codes (one 2-D TMA tile, 64 rows x 128 words = 32 KiB)
// and the stage's x' of each token (one bulk copy per token); all 32 lanes
// copy the fp16 scales and zeros of the unit's rows and groups (cp.async,
// counted on the same barrier).  Warps 0-15 each own 8 rows (row group
// warp % 8) and one half of the stage's columns (warp / 8); a lane takes 2
// code words of each row and the matching x' (16-byte, conflict-free
// shared-memory reads in the permuted order).  When a row block's segment
// ends, the column-half warp hands its sums to its row group's other warp
// through a 2-slot shared-memory exchange.  A row block finished inside one
// block is written to Y directly; one split across blocks leaves a partial
// sum per block, and the last block to arrive (counted per row block and row
// group) adds the partials in block order, so Y does not depend on timing.
// Partial slot of (row block rb, block b): rb + b, unique because both grow
// along the unit list.
template <int CB, int TT>
__global__ void __launch_bounds__(qlv::THREADS, 1)
qlinear_gemv_kernel(const __grid_constant__ CUtensorMap tmap_codes, const qlv::Args A) {
    using namespace qlv;
    constexpr int CPW = 32 / CB;                 // columns per word
    constexpr int SC = WORDS * CPW;              // columns per stage
    constexpr int V = RPW * TT;
    constexpr uint32_t TX_BYTES = CODE_BYTES + TT * SC * 4;
    const int gps = A.gps;
    const uint32_t STAGE_BYTES = stage_bytes(SC, TT, gps);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    float *pair_buf = reinterpret_cast<float *>(base + A.n_stages * STAGE_BYTES);
    uint64_t *full = reinterpret_cast<uint64_t *>(pair_buf + PAIR_FLOATS);
    uint64_t *empty = full + MAX_STAGES;
    uint64_t *pair_full = empty + MAX_STAGES;    // [RGROUPS][2]
    uint64_t *pair_empty = pair_full + 2 * RGROUPS;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t grid = gridDim.x;
    const int64_t u_begin = A.units * blockIdx.x / grid, u_end = A.units * (blockIdx.x + 1) / grid;
    if (threadIdx.x == 0) {
        // full: the producer's expect-tx arrive plus one cp.async arrive per lane
        for (int i = 0; i < A.n_stages; ++i) { mbar_init(&full[i], 33); mbar_init(&empty[i], CWARPS); }
        for (int i = 0; i < 2 * RGROUPS; ++i) { mbar_init(&pair_full[i], 1); mbar_init(&pair_empty[i], 1); }
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == CWARPS) {                        // producer
        if (lane == 0) tma_prefetch_desc(&tmap_codes);
        int st = 0;
        uint32_t ph = 0;
        int64_t rb = u_begin / A.n_steps, j = u_begin - rb * A.n_steps;
        const int per = A.sz_mode / 2;                   // groups per copy (16- or 4-byte modes)
        const int lcpr = __ffs(A.gps / per) - 1;          // log2(copies per row); gps and per are powers of 2
        static_assert(ROWS == 64, "copy indexing takes 6 bits for the row");
        for (int64_t u = u_begin; u < u_end; ++u, (++j == A.n_steps ? (j = 0, ++rb) : 0)) {
            if (!mbar_wait_warp(&empty[st], ph ^ 1u, &abort_flag, A.timeout_ns)) break;
            uint8_t *stage = base + st * STAGE_BYTES;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[st], TX_BYTES);
                tma_load_2d(stage, &tmap_codes, (int32_t)(j * WORDS), (int32_t)(rb * ROWS), &full[st]);
#pragma unroll
                for (int t = 0; t < TT; ++t)
                    bulk_load(stage + CODE_BYTES + t * SC * 4, A.xs + t * A.Kp + j * SC, SC * 4, &full[st]);
            }
            // scales then zeros of rows rb*64.. and groups j*gps.. (groups past G
            // belong to lanes past K, which never read them; rows past N repeat row N-1)
            __half *sz = reinterpret_cast<__half *>(stage + TX_BYTES);
            const int64_t g0 = j * gps;
            if (A.sz_mode == 2) {
                for (int e = lane; e < 2 * ROWS * gps; e += 32) {
                    const int arr = e / (ROWS * gps), rem = e % (ROWS * gps), r = rem / gps, g = rem % gps;
                    int64_t n = rb * ROWS + r;
                    n = n < A.N ? n : A.N - 1;
                    if (g0 + g < A.G) sz[e] = (arr ? A.zeros : A.scales)[n * A.G + g0 + g];
                }
                mbar_arrive(&full[st]);
            } else {
                for (int e = lane; e < (2 * ROWS) << lcpr; e += 32) {
                    const int arr = e >> (6 + lcpr), r = (e >> lcpr) & (ROWS - 1), c = e & ((1 << lcpr) - 1);
                    int64_t n = rb * ROWS + r;
                    n = n < A.N ? n : A.N - 1;
                    if (g0 + c * per >= A.G) continue;
                    const __half *src = (arr ? A.zeros : A.scales) + n * A.G + g0 + c * per;
                    __half *dst = sz + (arr * ROWS + r) * gps + c * per;
                    if (A.sz_mode == 16) cp_async_16(dst, src); else cp_async_4(dst, src);
                }
                cp_async_arrive_noinc(&full[st]);
            }
            if (++st == A.n_stages) { st = 0; ph ^= 1u; }
        }
    } else {                                     // consumers
        const int rg = warp % RGROUPS, hh = warp / RGROUPS;
        const int lane_col = hh * (SC / 2) + lane * 2 * CPW;     // first column of the lane in a stage
        const int gl = lane_col / A.group;                        // the lane's group within a stage
        float acc[RPW][TT];
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int t = 0; t < TT; ++t) acc[r][t] = 0.0f;
        int st = 0, ps = 0;
        uint32_t ph = 0, pph = 0;
        int64_t rb = u_begin / A.n_steps, j = u_begin - rb * A.n_steps - 1;
        for (int64_t u = u_begin; u < u_end; ++u) {
            if (++j == A.n_steps) { j = 0; ++rb; }
            if (!mbar_wait_warp(&full[st], ph, &abort_flag, A.timeout_ns)) break;
            const uint8_t *stage = base + st * STAGE_BYTES;
            if (j * SC + lane_col < A.K) {                       // lanes past K hold zero fill
                const __half *sz = reinterpret_cast<const __half *>(stage + TX_BYTES);
                float sh[RPW];
                float noff[RPW];                                 // -(2^23 + z)
#pragma unroll
                for (int r = 0; r < RPW; ++r) {
                    sh[r] = __half2float(sz[(rg * RPW + r) * gps + gl]);
                    noff[r] = -__fadd_rn(8388608.0f, __half2float(sz[(ROWS + rg * RPW + r) * gps + gl]));
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float x[TT][CPW];
#pragma unroll
                    for (int t = 0; t < TT; ++t)
#pragma unroll
                        for (int q = 0; q < CPW / 4; ++q) {
                            const float4 v = *reinterpret_cast<const float4 *>(
                                stage + CODE_BYTES + (t * SC + (((hh * 2 + i) * (CPW / 4) + q) * 32 + lane) * 4) * 4);
                            x[t][4 * q] = v.x; x[t][4 * q + 1] = v.y; x[t][4 * q + 2] = v.z; x[t][4 * q + 3] = v.w;
                        }
#pragma unroll
                    for (int r = 0; r < RPW; ++r) {
                        float d[CPW];
                        const uint32_t wr =
                            *reinterpret_cast<const uint32_t *>(stage + ((rg * RPW + r) * WORDS + hh * 64 + 2 * lane + i) * 4);
                        dequant_word<CB>(wr, make_float2(noff[r], noff[r]), d);
#pragma unroll
                        for (int t = 0; t < TT; ++t) {
                            float2 s2 = mul2_rn(make_float2(x[t][0], x[t][1]), make_float2(d[0], d[1]));
#pragma unroll
                            for (int e = 2; e < CPW; e += 2)
                                s2 = fma2_rn(make_float2(x[t][e], x[t][e + 1]), make_float2(d[e], d[e + 1]), s2);
                            acc[r][t] = __fmaf_rn(sh[r], __fadd_rn(s2.x, s2.y), acc[r][t]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);       // this warp is done with the stage
            if (++st == A.n_stages) { st = 0; ph ^= 1u; }
            if (j != A.n_steps - 1 && u != u_end - 1) continue;
            // ---- row block rb ends here (or this block's range does): flush ----
            float v[V];
#pragma unroll
            for (int r = 0; r < RPW; ++r)
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    v[r * TT + t] = acc[r][t];
                    acc[r][t] = 0.0f;
                }
            float mine = warp_reduce_scatter<V>(v);
            // the two column halves of the row group meet in shared memory
            float *slot = pair_buf + (rg * 2 + ps) * 32;
            if (hh == 1) {
                if (!mbar_wait_warp(&pair_empty[rg * 2 + ps], pph ^ 1u, &abort_flag, A.timeout_ns)) break;
                slot[lane] = mine;
                __syncwarp();
                if (lane == 0) mbar_arrive(&pair_full[rg * 2 + ps]);
                if (++ps == 2) { ps = 0; pph ^= 1u; }
                continue;
            }
            if (!mbar_wait_warp(&pair_full[rg * 2 + ps], pph, &abort_flag, A.timeout_ns)) break;
            mine = __fadd_rn(mine, slot[lane]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&pair_empty[rg * 2 + ps]);
            if (++ps == 2) { ps = 0; pph ^= 1u; }
            const int r = (lane % V) / TT, t = lane % TT;
            const int64_t n = rb * ROWS + rg * RPW + r;
            const bool writer = lane < V && n < A.N && t < A.T;
            const int64_t rb_u0 = rb * A.n_steps, rb_u1 = rb_u0 + A.n_steps;
            if (u_begin <= rb_u0 && u_end >= rb_u1) {       // whole row block in this block
                if (writer) A.Y[t * A.N + n] = mine;
                continue;
            }
            A.part[(rb + blockIdx.x) * SLOT_FLOATS + rg * 32 + lane] = mine;
            __threadfence();
            __syncwarp();
            const int64_t b0 = block_of(rb_u0, A.units, grid), b1 = block_of(rb_u1 - 1, A.units, grid);
            unsigned old = 0;
            if (lane == 0) old = atomicAdd(&A.cnt[rb * RGROUPS + rg], 1u);
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old != (unsigned)(b1 - b0)) continue;
            __threadfence();                              // last to arrive: sum the partials in block order
            float y = 0.0f;
            for (int64_t b = b0; b <= b1; ++b) y = __fadd_rn(y, __ldcg(&A.part[(rb + b) * SLOT_FLOATS + rg * 32 + lane]));
            if (writer) A.Y[t * A.N + n] = y;
            if (lane == 0) A.cnt[rb * RGROUPS + rg] = 0u;    // ready for the next launch
        }
    }
    // copies issued by the producer land before the block can leave
    if (abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    __syncthreads();
}

// ===========================================================================
// The decode consumer on the tensor cores ([AWQ-note] "Tiny Chat": the codes are
// dequantized inside the kernel), any w_bit.  The same definition as the
// CUDA-core kernel,
//   Y[t, n] = sum_k x'[t, k] (q[n, k] - z[n, g]) sh[n, g],   x' = RN32(x RN32(1/s)),
// evaluated as Y = sum_g sh (D_g - z S_g) with
//   D_g[n, t] = sum_{k in g} q[n, k] x'[t, k]   on tcgen05 (kind::f16, bf16 operands, fp32 accumulate),
//   S_g[t]    = RN32(sum_{k in g} x'[t, k])     in binary64 by qtc_prep_kernel.
// Both MMA operands hold exact values: A = q (an integer below 16, exact in
// bf16) and B = x' split into three bf16 pieces whose sum is x' exactly
// (8 + 8 + 8 significant bits), one B row per piece and token.  So every
// product the tensor core forms is exact and only the fp32 accumulation
// rounds; no step depends on the range of the zero point.  The work layout and
// the roles of the warps are described at qlinear_tc_kernel.
// ===========================================================================

// The 8 codes of one 8-column chunk (code e in bits CB e .. of x) as 4 bf16x2
// words of A: word e holds (code e, code e + 4).  One mask places the two codes
// in the two halves under the bf16 exponent of 128, one bf16x2 subtraction of
// 128 leaves them exactly.  The B operand's columns follow the same order
// (column 2e of the chunk is x' of column e, column 2e + 1 that of e + 4).
template <int CB>
__device__ __forceinline__ void qtc_chunk_bf16(uint32_t x, uint32_t *v) {
    const __nv_bfloat162 off = __floats2bfloat162_rn(128.0f, 128.0f);
    constexpr uint32_t mask = CB == 4 ? 0x000F000Fu : 0x00030003u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t u = ((x >> (CB * e)) & mask) | 0x43004300u;
        const __nv_bfloat162 b = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&u), off);
        v[e] = *reinterpret_cast<const uint32_t *>(&b);
    }
}

namespace qtc {
constexpr int ROWS = 128;                 // W rows per unit (MMA M)
constexpr int SC = 256;                   // K columns per unit: 16 MMAs of K 16
constexpr int A_COLS = SC / 2;            // tensor-memory columns of one A slot (2 bf16 per column)
constexpr int TMEM_COLS = 512;
constexpr int CODE_BYTES = ROWS * 128;    // one unit's codes: 128 (4-bit) or 64 (2-bit) bytes a row
constexpr int TT_MAX = 16;
constexpr int SLOT_FLOATS = ROWS * TT_MAX;                    // one partial-sum slot: 128 rows x 16 tokens
constexpr int PWARPS = 8;                 // producers: lane quadrant warp % 4, column half warp / 4
constexpr int EWARP0 = 8;                 // epilogue: warps 8-11, lane quadrant warp - 8, one row per thread
constexpr int MMA_WARP = 12, LOAD_WARP = 13, BLOAD_WARP = 14, MMA_WARP2 = 15;   // MMA issue (two warps); code loads; B loads
constexpr int THREADS = 16 * 32;
// Token tiles: N = 16, 32 or 48 rows of x' pieces per pass (5, 10 or 16 tokens).
__host__ __device__ constexpr int tile_tokens(int nr) { return nr == 16 ? 5 : nr == 32 ? 10 : 16; }
template <int NR> __host__ __device__ constexpr int b_bytes() { return NR * SC * 2; }   // 4 swizzled boxes of NR x 64
// Two rings: code tiles, freed once the producers have converted them, deep
// enough to cover the load latency of HBM under load; B tiles, freed when the
// MMAs that read them complete.
template <int NR> __host__ __device__ constexpr int code_stages() { return NR == 16 ? 10 : NR == 32 ? 8 : 7; }
constexpr int B_STAGES = 4;
// Accumulator columns of one unit: one NR-wide block per group of the unit.
template <int NR, int GPS> __host__ __device__ constexpr int d_cols() { return GPS * NR; }
template <int NR, int GPS> __host__ __device__ constexpr int a_slots() {
    return 3 * A_COLS + 2 * d_cols<NR, GPS>() <= TMEM_COLS ? 3 : 2;
}
template <int NR, int GPS> __host__ __device__ constexpr int d_bufs() {
    return (TMEM_COLS - a_slots<NR, GPS>() * A_COLS) / d_cols<NR, GPS>() > 4
               ? 4
               : (TMEM_COLS - a_slots<NR, GPS>() * A_COLS) / d_cols<NR, GPS>();
}
// Group sums S of the epilogue: per epilogue warp, two slots of 4 groups x 16 tokens.
constexpr int S_AREA_BYTES = 4 * 2 * 64 * 4;
template <int NR> constexpr size_t smem_bytes() {
    return (size_t)code_stages<NR>() * CODE_BYTES + (size_t)B_STAGES * b_bytes<NR>() + 1024 + 512 + S_AREA_BYTES;
}
static_assert(smem_bytes<16>() <= 232448 && smem_bytes<32>() <= 232448 && smem_bytes<48>() <= 232448,
              "decode shared memory above the 227 KiB a CTA may use");
// The block whose unit range [units*b/grid, units*(b+1)/grid) holds unit u.
__device__ __forceinline__ int64_t block_of(int64_t u, int64_t units, int64_t grid) {
    return ((u + 1) * grid - 1) / units;
}
// word i (0..4 NCH - 1) of NCH 16-byte chunks, i known at compile time
template <int NCH>
__device__ __forceinline__ uint32_t word_of(const uint4 (&cw)[NCH], int i) {
    const uint4 c = cw[i >> 2];
    return (i & 3) == 0 ? c.x : (i & 3) == 1 ? c.y : (i & 3) == 2 ? c.z : c.w;
}
// fp16 value o (0..7) of eight packed in 16 bytes
__device__ __forceinline__ float half_at(const uint4 &v, int o) {
    const uint32_t w = (o >> 1) == 0 ? v.x : (o >> 1) == 1 ? v.y : (o >> 1) == 2 ? v.z : v.w;
    return __half2float(__ushort_as_half((unsigned short)((o & 1) ? (w >> 16) : (w & 0xFFFFu))));
}
// One row's fp16 values by group ([N][G] scales or zeros) for the units a block
// walks through in order.  With G a multiple of 8 the thread reads 8 groups (16
// bytes) at a time, one chunk ahead of use; otherwise one value per group at use.
template <int GPS>
struct RowGroups {
    const __half *p;
    int64_t N, n_steps;
    int G, rr;
    bool vec;
    uint4 cur, nxt;
    int64_t nrb;                          // chunk held in nxt: row block, chunk index
    int nc;
    __device__ __forceinline__ uint4 fetch(int64_t rb, int c) const {
        int64_t n = rb * ROWS + rr;
        n = n < N ? n : N - 1;
        return __ldg(reinterpret_cast<const uint4 *>(p + n * G) + c);
    }
    // the chunk after (nrb, nc): a row block's chunks end at its n_steps * GPS
    // groups (= G when G is a multiple of 8, since K is then a multiple of 256)
    __device__ __forceinline__ void next_chunk() {
        if ((int64_t)(nc + 1) * 8 < n_steps * GPS) {
            ++nc;
        } else {
            ++nrb;
            nc = 0;
        }
    }
    __device__ __forceinline__ void begin(int64_t rb, int64_t j) {
        vec = G % 8 == 0;
        if (vec) {
            nrb = rb;
            nc = (int)((j * GPS) >> 3);
            cur = fetch(nrb, nc);
            next_chunk();
            nxt = fetch(nrb, nc);
        }
    }
    // called on reaching unit (., j), for every unit after the first
    __device__ __forceinline__ void enter(int64_t j) {
        if (vec && ((j * GPS) & 7) == 0) {
            cur = nxt;
            next_chunk();
            nxt = fetch(nrb, nc);
        }
    }
    __device__ __forceinline__ float get(int64_t rb, int64_t j, int g) const {
        const int64_t gg = j * GPS + g;
        if (vec) return half_at(cur, (int)(gg & 7));
        int64_t n = rb * ROWS + rr;
        n = n < N ? n : N - 1;
        return __half2float(__ldg(p + n * G + gg));
    }
};
struct Args {
    const __half *scales, *zeros;          // [N][G]
    const float *gsum;                     // S of this pass: [G][16]
    int64_t N;
    int G, T;                              // groups per row; tokens of this pass (<= TT)
    int64_t n_steps, units;                // units per row block (K / 256, rounded up); row blocks x n_steps
    int32_t b_row0;                        // first B row of this pass in the B map
    float *Y;                              // this pass's output rows [T][N]
    float *part;                           // partial sums of split row blocks: [(row blocks + grid) * 128][16]
    unsigned *cnt;                         // arrivals per row block and lane quadrant [row blocks][4]
    uint64_t timeout_ns;
};
}  // namespace qtc

// The operands the main kernel reads besides the codes, in one launch:
//   xb: x' = RN32(x RN32(1/s)) split into three bf16 pieces, stored as the B rows
//       of every pass: row piece * TT + t of pass p holds piece `piece` of token
//       p TT + t; within each 8-column chunk column c holds x' of column
//       (c / 2) + 4 (c % 2), the order of A's codes (qtc_chunk_bf16); rows past
//       3 TT, tokens past T and columns past K are zero;
//   gsum: S[p][g][t] = RN32(sum over the group's columns of x'[p TT + t, k]) in
//       binary64 (16 slots per group; tokens past the pass or past T give 0).  16
//       lanes per value: lane j sums columns j * group/16 .. + group/16 - 1, then
//       the 16 partial sums are added by shuffles (that loop's thread count is a
//       multiple of 32, and so is the grid's);
//   cnt: the main kernel's arrival counters, cleared.
// The main kernel may start early (programmatic dependent launch): its roles
// that read these wait for this grid with griddepcontrol.wait.
__global__ void qtc_prep_kernel(const __half *__restrict__ X, int64_t T, int64_t K, int64_t Kp, int64_t ldx,
                                const float *__restrict__ s, int TT, int NR, int n_pass, int G, int group,
                                __nv_bfloat16 *__restrict__ xb, float *__restrict__ gsum,
                                unsigned *__restrict__ cnt, int64_t n_cnt) {
    griddep_launch_dependents();
    const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, nth = (int64_t)gridDim.x * blockDim.x;
    const int64_t total = (int64_t)n_pass * NR * Kp;
    for (int64_t i = tid; i < total; i += nth) {
        const int64_t kb = i % Kp, rowg = i / Kp;
        const int64_t k = (kb & ~int64_t(7)) + ((kb & 7) >> 1) + 4 * (kb & 1);
        const int row = (int)(rowg % NR), pass = (int)(rowg / NR);
        const int piece = row / TT, t = row % TT;
        const int64_t tok = (int64_t)pass * TT + t;
        float v = 0.0f;
        if (piece < 3 && tok < T && k < K) {
            const float xp = __fmul_rn(__half2float(X[tok * ldx + k]), __frcp_rn(s[k]));
            const __nv_bfloat16 h = __float2bfloat16_rn(xp);
            const float r1 = __fsub_rn(xp, __bfloat162float(h));                 // exact
            const __nv_bfloat16 m = __float2bfloat16_rn(r1);
            const float r2 = __fsub_rn(r1, __bfloat162float(m));                 // exact, <= 8 bits
            v = piece == 0 ? __bfloat162float(h) : piece == 1 ? __bfloat162float(m) : r2;
        }
        xb[i] = __float2bfloat16_rn(v);                                          // exact for every piece
    }
    const int64_t gtotal = (int64_t)n_pass * G * 16 * 16;
    const int per = group / 16;
    for (int64_t i = tid; i < gtotal; i += nth) {
        const int j = (int)(i & 15);
        const int64_t o = i >> 4;
        const int t = (int)(o % 16);
        const int64_t pg = o / 16;
        const int g = (int)(pg % G), pass = (int)(pg / G);
        const int64_t tok = (int64_t)pass * TT + t;
        double acc = 0.0;
        if (t < TT && tok < T) {
            const int64_t kb = (int64_t)g * group + (int64_t)j * per;
            for (int c = 0; c < per; ++c)
                acc = __dadd_rn(acc, (double)__fmul_rn(__half2float(X[tok * ldx + kb + c]), __frcp_rn(s[kb + c])));
        }
#pragma unroll
        for (int o2 = 8; o2 >= 1; o2 >>= 1) acc = __dadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o2));
        if (j == 0) gsum[o] = __double2float_rn(acc);
    }
    for (int64_t i = tid; i < n_cnt; i += nth) cnt[i] = 0u;
}

// One pass (up to TT tokens) of the packed layer on the tensor cores.  Persistent:
// block b takes the contiguous units [units b / grid, units (b + 1) / grid) of the
// list (row block of 128 rows, step of 256 columns), row-block major, so every
// block streams the same number of code bytes.  Roles:
//   warp 13: the codes, one 2-D TMA tile per unit (128 rows x 128 or 64 bytes,
//            swizzled), into a ring of code_stages tiles;
//   warp 14: the unit's B tile, 4 boxes of NR x 64 bf16 (128-byte swizzle);
//   warps 0-7: producers; warp w converts columns 128 (w / 4) .. + 127 of the rows
//            of lane quadrant w % 4 (one row per thread) into A slot as of tensor
//            memory with tcgen05.st, then releases the code tile;
//   warps 12 and 15: one thread each issues the 16 MMAs of every other unit (A
//            from tensor memory, B from shared memory) into one accumulator per
//            group, then commits;
//   warps 8-11: epilogue; each thread drains its row's accumulators, applies
//            sh (D - z S) and, at the end of its row block's segment, writes Y or
//            a partial sum that the last block to arrive adds in block order.
template <int NR, int CB, int GPS>
__global__ void __launch_bounds__(qtc::THREADS, 1)
qlinear_tc_kernel(const __grid_constant__ CUtensorMap tmap_codes, const __grid_constant__ CUtensorMap tmap_b,
                  const qtc::Args A) {
    using namespace qtc;
    constexpr int CS = code_stages<NR>();
    constexpr int BS = B_STAGES;
    constexpr int D_COLS = d_cols<NR, GPS>();
    constexpr int AS = a_slots<NR, GPS>();         // A slots in tensor memory
    constexpr int DB = d_bufs<NR, GPS>();          // accumulator buffers
    constexpr int MPG = 16 / GPS;                  // MMAs (K 16 each) per group
    // Issuing threads.  A thread that takes every other unit waits on an
    // accumulator buffer's d_empty for every other release of it; its parity
    // wait is unambiguous only if the buffer ring holds two or more buffers.
    constexpr int NISSUE = DB >= 2 ? 2 : 1;
    constexpr int TT = tile_tokens(NR);
    constexpr int NCH = CB == 4 ? 4 : 2;           // 16-byte code chunks of a producer thread per unit
    static_assert(AS * A_COLS + DB * D_COLS <= TMEM_COLS && DB >= 1, "tensor memory budget");
    static_assert(3 * TT <= NR, "three pieces per token");
    constexpr uint32_t IDESC = mma_idesc_bf16_f32(ROWS, NR);
    constexpr uint32_t B_BYTES = b_bytes<NR>();
    constexpr uint32_t CODE_TX = ROWS * (CB == 4 ? 128 : 64);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *bring = base + CS * CODE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(bring + BS * B_BYTES);
    uint64_t *full = bars, *empty = bars + CS, *b_full = bars + 2 * CS, *b_empty = b_full + BS;
    uint64_t *a_full = b_empty + BS, *a_empty = a_full + AS, *d_full = a_empty + AS, *d_empty = d_full + DB;
    uint64_t *drain = d_empty + DB;                // one per issuing thread
    static_assert((2 * CS + 2 * BS + 2 * AS + 2 * DB + 2) * 8 <= 512, "barrier area");
    float *s_area = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + 512);
    __shared__ uint32_t tmem_base_sm;
    __shared__ int abort_sm;
    volatile int *abort_flag = &abort_sm;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t grid = gridDim.x;
    const int64_t u_begin = A.units * blockIdx.x / grid, u_end = A.units * (blockIdx.x + 1) / grid;
    if (threadIdx.x == 0) {
        for (int i = 0; i < CS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], PWARPS); }
        for (int i = 0; i < BS; ++i) { mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < AS; ++i) { mbar_init(&a_full[i], PWARPS); mbar_init(&a_empty[i], 1); }
        for (int i = 0; i < DB; ++i) { mbar_init(&d_full[i], 1); mbar_init(&d_empty[i], 4); }
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        abort_sm = 0;
        fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc_1(&tmem_base_sm, TMEM_COLS);
        tmem_relinquish_1();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sm;
    bool aborted = false;

    if (warp == LOAD_WARP) {                       // code tiles (TMA)
        if (lane == 0) {
            tma_prefetch_desc(&tmap_codes);
            int st = 0;
            uint32_t ph = 0;
            int64_t rb = u_begin / A.n_steps, j = u_begin - rb * A.n_steps;
            for (int64_t u = u_begin; u < u_end; ++u) {
                if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, A.timeout_ns)) { aborted = true; break; }
                mbar_arrive_expect_tx(&full[st], CODE_TX);
                tma_load_2d(base + st * CODE_BYTES, &tmap_codes, (int32_t)(j * (SC * CB / 32)), (int32_t)(rb * ROWS),
                            &full[st]);
                if (++st == CS) { st = 0; ph ^= 1u; }
                if (++j == A.n_steps) { j = 0; ++rb; }
            }
        }
    } else if (warp == BLOAD_WARP) {               // x' pieces of the unit's 256 columns (TMA)
        if (lane == 0) {
            tma_prefetch_desc(&tmap_b);
            griddep_wait();                        // x' pieces written by the prep grid
            int st = 0;
            uint32_t ph = 0;
            int64_t j = u_begin % A.n_steps;
            for (int64_t u = u_begin; u < u_end; ++u) {
                if (!mbar_wait_bounded(&b_empty[st], ph ^ 1u, abort_flag, A.timeout_ns)) { aborted = true; break; }
                uint8_t *bst = bring + st * B_BYTES;
                mbar_arrive_expect_tx(&b_full[st], B_BYTES);
#pragma unroll
                for (int a = 0; a < 4; ++a)
                    tma_load_2d(bst + a * NR * 128, &tmap_b, (int32_t)(j * SC + a * 64), A.b_row0, &b_full[st]);
                if (++st == BS) { st = 0; ph ^= 1u; }
                if (++j == A.n_steps) j = 0;
            }
        }
    } else if (warp == MMA_WARP || warp == MMA_WARP2) {   // two threads issue the MMAs, units in turn
        if (lane == 0) {
            // thread mt takes the units u_begin + mt, u_begin + mt + NISSUE, ...: each
            // unit's MMAs come from one thread in order, and the two threads' issue
            // latencies overlap.  Both follow every unit's slots and phases.
            const int mt = warp == MMA_WARP ? 0 : 1;
            int bs = 0, as = 0, db = 0;
            uint32_t bph = 0, aph = 0, dph = 0;
            for (int64_t u = u_begin; u < u_end && mt < NISSUE; ++u) {
                if ((int)((u - u_begin) % NISSUE) == mt) {
                    if (!mbar_wait_bounded(&b_full[bs], bph, abort_flag, A.timeout_ns) ||
                        !mbar_wait_bounded(&a_full[as], aph, abort_flag, A.timeout_ns) ||
                        !mbar_wait_bounded(&d_empty[db], dph ^ 1u, abort_flag, A.timeout_ns)) { aborted = true; break; }
                    tc_fence_after();
                    // every offset below is a compile-time constant: the descriptor's start
                    // address field (address / 16) takes the byte offset / 16 directly
                    const uint64_t bd0 = sw128_kmajor_desc(smem_u32(bring + bs * B_BYTES));
                    const uint32_t d0 = tmem + AS * A_COLS + db * D_COLS, a0 = tmem + as * A_COLS;
#pragma unroll
                    for (int m = 0; m < SC / 16; ++m)
                        mma_f16_ts(d0 + (m / MPG) * NR, a0 + 8 * m,
                                   bd0 + (uint64_t)(((m / 4) * NR * 128 + (m % 4) * 32) >> 4), IDESC, m % MPG != 0);
                    mma_commit_1(&a_empty[as]);
                    mma_commit_1(&b_empty[bs]);
                    mma_commit_1(&d_full[db]);
                }
                if (++bs == BS) { bs = 0; bph ^= 1u; }
                if (++as == AS) { as = 0; aph ^= 1u; }
                if (++db == DB) { db = 0; dph ^= 1u; }
            }
            mma_commit_1(&drain[mt]);              // every MMA this thread issued has finished when this fires
            mbar_wait_bounded(&drain[mt], 0, abort_flag, A.timeout_ns);
        }
    } else if (warp < PWARPS) {                    // producers: A = q as bf16 pairs
        const int q = warp & 3, h = warp >> 2;
        const int rr = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int st = 0, as = 0;
        uint32_t ph = 0, aph = 0;
        for (int64_t u = u_begin; u < u_end; ++u) {
            if (!mbar_wait_warp(&full[st], ph, abort_flag, A.timeout_ns)) { aborted = true; break; }
            const uint8_t *stage = base + st * CODE_BYTES;
            uint4 cw[NCH];
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                // 4-bit: 128-byte rows, 128-byte swizzle; 2-bit: 64-byte rows, 64-byte swizzle
                const uint32_t off = CB == 4 ? (uint32_t)rr * 128u + ((uint32_t)((4 * h + c) ^ (rr & 7)) << 4)
                                             : (uint32_t)rr * 64u + ((uint32_t)((2 * h + c) ^ ((rr >> 1) & 3)) << 4);
                cw[c] = *reinterpret_cast<const uint4 *>(stage + off);
            }
            if (!mbar_wait_warp(&a_empty[as], aph ^ 1u, abort_flag, A.timeout_ns)) { aborted = true; break; }
            tc_fence_after();
#pragma unroll
            for (int half8 = 0; half8 < 2; ++half8) {  // 64 columns: tensor-memory columns 64 h + 32 half8 ..
                uint32_t v[32];
                if (CB == 4) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) qtc_chunk_bf16<4>(word_of<NCH>(cw, half8 * 8 + i), &v[4 * i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t w = word_of<NCH>(cw, half8 * 4 + i);   // 16 codes: two chunks
                        qtc_chunk_bf16<2>(__byte_perm(w, 0u, 0x4140u), &v[8 * i]);
                        qtc_chunk_bf16<2>(__byte_perm(w, 0u, 0x4342u), &v[8 * i + 4]);
                    }
                }
                tmem_st_32x32b_x32(tmem + lane_base + (uint32_t)(as * A_COLS + 64 * h + 32 * half8), v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&a_full[as]);
                // the code tile is released only now that the conversion has consumed
                // every value read from it: a load is complete once an instruction has
                // read its register, so an arrive right after the loads could let the
                // next tile's copy overwrite the stage under a load still in flight
                mbar_arrive(&empty[st]);
            }
            if (++as == AS) { as = 0; aph ^= 1u; }
            if (++st == CS) { st = 0; ph ^= 1u; }
        }
    } else if (warp >= EWARP0 && warp < EWARP0 + 4) {   // epilogue: one row per thread
        const int q = warp - EWARP0;
        const int rr = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        griddep_wait();                            // group sums and counters written by the prep grid
        float y[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) y[t] = 0.0f;
        int db = 0;
        uint32_t dph = 0;
        int64_t rb = u_begin / A.n_steps, j = u_begin - rb * A.n_steps;
        RowGroups<GPS> sr{A.scales, A.N, A.n_steps, A.G, rr}, zr{A.zeros, A.N, A.n_steps, A.G, rr};
        if (u_begin < u_end) {
            sr.begin(rb, j);
            zr.begin(rb, j);
        }
        // The unit's group sums S_g[t] (the same for every row) through this warp's
        // two shared-memory slots of 64 values (group e / 16, token slot e % 16):
        // lane l loads values l and l + 32 of the unit two ahead into registers and
        // stores them one unit later, so no load latency sits on a unit.
        float *sw = s_area + q * 128;
        auto s_load = [&](int64_t jj, float &v0, float &v1) {
            const int g0 = lane >> 4, g1 = 2 + (lane >> 4);
            const int64_t a0 = jj * GPS + g0, a1 = jj * GPS + g1;
            v0 = (g0 < GPS && a0 < A.G) ? __ldg(A.gsum + a0 * 16 + (lane & 15)) : 0.0f;
            v1 = (g1 < GPS && a1 < A.G) ? __ldg(A.gsum + a1 * 16 + (lane & 15)) : 0.0f;
        };
        auto next_step = [&](int64_t jj) { return jj + 1 == A.n_steps ? int64_t(0) : jj + 1; };
        int64_t j_next = next_step(j), j_next2 = next_step(j_next);   // steps of the next two units
        float p0 = 0.0f, p1 = 0.0f;
        if (u_begin < u_end) {
            float c0, c1;
            s_load(j, c0, c1);
            sw[lane] = c0;
            sw[lane + 32] = c1;
            s_load(j_next, p0, p1);
        }
        for (int64_t u = u_begin; u < u_end; ++u) {
            const int slot = (int)((u - u_begin) & 1);
            __syncwarp();                          // every lane is done with the other slot
            if (u + 1 < u_end) {
                sw[(slot ^ 1) * 64 + lane] = p0;
                sw[(slot ^ 1) * 64 + lane + 32] = p1;
            }
            if (u + 2 < u_end) s_load(j_next2, p0, p1);
            __syncwarp();                          // this unit's slot is complete
            const float *su = sw + slot * 64;
            j_next = j_next2;
            j_next2 = next_step(j_next2);
            if (u != u_begin) {
                sr.enter(j);
                zr.enter(j);
            }
            if (!mbar_wait_warp(&d_full[db], dph, abort_flag, A.timeout_ns)) { aborted = true; break; }
            tc_fence_after();
            const uint32_t dbase = tmem + lane_base + (uint32_t)(AS * A_COLS + db * D_COLS);
            if constexpr (D_COLS == 32) {
                // the whole unit's accumulators (two groups of 16 columns) in one load
                // and one wait; the buffer is released before the arithmetic (a
                // 64-column load measured slower, so wider units take the path below)
                float dv[D_COLS];
                tmem_ld_32x32b_x32_sync(dbase, dv);
                tc_fence_before();
                __syncwarp();                      // every lane's reads are complete (wait::ld)
                if (lane == 0) mbar_arrive(&d_empty[db]);
#pragma unroll
                for (int g = 0; g < GPS; ++g) {
                    const int64_t gg = j * GPS + g;
                    if (gg < A.G) {                // past G the codes and x' are zero: no term
                        const float shg = sr.get(rb, j, g), zg = zr.get(rb, j, g);
#pragma unroll
                        for (int t = 0; t < TT; ++t) {
                            // (hi + mid) + lo: accumulator columns t, TT + t, 2 TT + t of the group
                            const float dt = __fadd_rn(__fadd_rn(dv[g * NR + t], dv[g * NR + TT + t]), dv[g * NR + 2 * TT + t]);
                            y[t] = __fmaf_rn(shg, __fmaf_rn(-zg, su[g * 16 + t], dt), y[t]);
                        }
                    }
                }
            } else {
#pragma unroll
                for (int g = 0; g < GPS; ++g) {
                    // dt[t] = (hi + mid) + lo: accumulator columns t, TT + t, 2 TT + t
                    float dt[TT];
                    const uint32_t dcol = dbase + (uint32_t)(g * NR);
                    if constexpr (NR == 48) {      // TT = 16: one 16-column load per piece
                        float pc[16];
                        tmem_ld_32x32b_x16_sync(dcol, pc);
#pragma unroll
                        for (int t = 0; t < TT; ++t) dt[t] = pc[t];
                        tmem_ld_32x32b_x16_sync(dcol + 16, pc);
#pragma unroll
                        for (int t = 0; t < TT; ++t) dt[t] = __fadd_rn(dt[t], pc[t]);
                        tmem_ld_32x32b_x16_sync(dcol + 32, pc);
#pragma unroll
                        for (int t = 0; t < TT; ++t) dt[t] = __fadd_rn(dt[t], pc[t]);
                    } else {
                        float dv[NR];
#pragma unroll
                        for (int c = 0; c < NR; c += 16)
                            tmem_ld_32x32b_x16_sync(dcol + c, *reinterpret_cast<float(*)[16]>(&dv[c]));
#pragma unroll
                        for (int t = 0; t < TT; ++t) dt[t] = __fadd_rn(__fadd_rn(dv[t], dv[TT + t]), dv[2 * TT + t]);
                    }
                    const int64_t gg = j * GPS + g;
                    if (gg < A.G) {                // past G the codes and x' are zero: no term
                        const float shg = sr.get(rb, j, g), zg = zr.get(rb, j, g);
#pragma unroll
                        for (int t = 0; t < TT; ++t) y[t] = __fmaf_rn(shg, __fmaf_rn(-zg, su[g * 16 + t], dt[t]), y[t]);
                    }
                }
                tc_fence_before();
                __syncwarp();                      // every lane's reads are complete (wait::ld)
                if (lane == 0) mbar_arrive(&d_empty[db]);
            }
            if (++db == DB) { db = 0; dph ^= 1u; }
            if (j == A.n_steps - 1 || u == u_end - 1) {
                // row block rb's segment ends: Y, or a partial sum and the fixup
                const int64_t n = rb * ROWS + rr;
                const int64_t rb_u0 = rb * A.n_steps, rb_u1 = rb_u0 + A.n_steps;
                if (u_begin <= rb_u0 && u_end >= rb_u1) {
                    if (n < A.N)
#pragma unroll
                        for (int t = 0; t < TT; ++t)
                            if (t < A.T) A.Y[t * A.N + n] = y[t];
                } else {
                    float *mine = A.part + ((rb + blockIdx.x) * ROWS + rr) * TT_MAX;
#pragma unroll
                    for (int t = 0; t < TT; ++t) mine[t] = y[t];
                    __threadfence();
                    __syncwarp();
                    const int64_t b0 = block_of(rb_u0, A.units, grid), b1 = block_of(rb_u1 - 1, A.units, grid);
                    unsigned old = 0;
                    if (lane == 0) old = atomicAdd(&A.cnt[rb * 4 + q], 1u);
                    old = __shfl_sync(0xffffffffu, old, 0);
                    if (old == (unsigned)(b1 - b0)) {
                        __threadfence();
                        float tot[TT];
#pragma unroll
                        for (int t = 0; t < TT; ++t) tot[t] = 0.0f;
                        for (int64_t b = b0; b <= b1; ++b)
#pragma unroll
                            for (int t = 0; t < TT; ++t)
                                tot[t] = __fadd_rn(tot[t], __ldcg(A.part + ((rb + b) * ROWS + rr) * TT_MAX + t));
                        if (n < A.N)
#pragma unroll
                            for (int t = 0; t < TT; ++t)
                                if (t < A.T) A.Y[t * A.N + n] = tot[t];
                        if (lane == 0) A.cnt[rb * 4 + q] = 0u;
                    }
                }
#pragma unroll
                for (int t = 0; t < TT; ++t) y[t] = 0.0f;
            }
            if (++j == A.n_steps) {
                j = 0;
                ++rb;
            }
        }
    }

    if (aborted || *abort_flag) {                  // let copies in flight land before the block exits
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_1(tmem, TMEM_COLS);
    }
}

// ===========================================================================
// AWQ followed by GPTQ error compensation ([AWQ-note] "Measures": AWQ+GPTQ;
// [Notes-52] §4: round a column, push its error into the columns not yet
// quantized, weighted by second-order statistics of the real input;
// [GPTQ-AWQ] "GPTQ": a column sweep with a Cholesky factor prepared once).
//   H  = 2 X'^T X',  x' = RN32(x RN32(1/s))                 (gptq_hessian_kernel)
//   Hd = H + damp mean(diag H) I;  U upper with Hd^-1 = U^T U (gptq_* factor kernels)
//   per row, in binary32: the column sweep                   (gptq_sweep_kernel)
// All in binary32.  The factor: with P the order-reversing permutation,
// A = P Hd P = L L^T (lower Cholesky), so Hd = R R^T with R = P L P upper and
// Hd^-1 = (R^-1)^T R^-1: U = R^-1 = P L^-1 P, the 180-degree rotation of L^-1.
// ===========================================================================
constexpr int kGb = 64;                  // block size of the factor kernels and the Hessian tile

// Index (bi, bj), bi >= bj, of the t-th block of a lower block triangle, rows first.
__device__ __forceinline__ void lower_block(int t, int &bi, int &bj) {
    int i = (int)((sqrtf(8.0f * (float)t + 1.0f) - 1.0f) * 0.5f);
    while ((i + 1) * (i + 2) / 2 <= t) ++i;
    while (i * (i + 1) / 2 > t) --i;
    bi = i;
    bj = t - i * (i + 1) / 2;
}

// H tile (bi, bj), bi >= bj, of 64 x 64: each thread a 4 x 4 patch, the
// tokens in order (binary32 FMA), 16 tokens per shared-memory stage; the
// tile and its mirror are written.
__global__ void __launch_bounds__(256)
gptq_hessian_kernel(const __half *__restrict__ X, int64_t T, int64_t K, int64_t ldx, const float *__restrict__ s,
                    float *__restrict__ H) {
    __shared__ __align__(16) float xi[16][kGb + 4];
    __shared__ __align__(16) float xj[16][kGb + 4];
    int bi, bj;
    lower_block(blockIdx.x, bi, bj);
    const int64_t i0 = (int64_t)bi * kGb, j0 = (int64_t)bj * kGb;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int lr = threadIdx.x / 16, lc = (threadIdx.x % 16) * 4;   // loader: token row, 4 columns
    float rsi[4], rsj[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        rsi[e] = __frcp_rn(s[i0 + lc + e]);
        rsj[e] = __frcp_rn(s[j0 + lc + e]);
    }
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
    for (int64_t t0 = 0; t0 < T; t0 += 16) {
        const int64_t t = t0 + lr;
        float vi[4] = {0.0f, 0.0f, 0.0f, 0.0f}, vj[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (t < T) {
            const uint2 hi = *reinterpret_cast<const uint2 *>(X + t * ldx + i0 + lc);
            const uint2 hj = *reinterpret_cast<const uint2 *>(X + t * ldx + j0 + lc);
            const __half *pi = reinterpret_cast<const __half *>(&hi);
            const __half *pj = reinterpret_cast<const __half *>(&hj);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                vi[e] = __fmul_rn(__half2float(pi[e]), rsi[e]);
                vj[e] = __fmul_rn(__half2float(pj[e]), rsj[e]);
            }
        }
        __syncthreads();
        *reinterpret_cast<float4 *>(&xi[lr][lc]) = make_float4(vi[0], vi[1], vi[2], vi[3]);
        *reinterpret_cast<float4 *>(&xj[lr][lc]) = make_float4(vj[0], vj[1], vj[2], vj[3]);
        __syncthreads();
#pragma unroll
        for (int tt = 0; tt < 16; ++tt) {
            const float4 a = *reinterpret_cast<const float4 *>(&xi[tt][ty * 4]);
            const float4 b = *reinterpret_cast<const float4 *>(&xj[tt][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[p][q] = __fmaf_rn(av[p], bv[q], acc[p][q]);
        }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t i = i0 + ty * 4 + p, j = j0 + tx * 4 + q;
            const float v = __fmul_rn(2.0f, acc[p][q]);
            H[i * K + j] = v;
            if (bi != bj) H[j * K + i] = v;
        }
}

// H = 2 X'^T X' on the tensor cores.  x' = RN32(x RN32(1/s)) is split into
// three bf16 pieces whose sum is x' exactly (hi = RN(x'), mid = RN(x' - hi),
// lo = x' - hi - mid), so every product of pieces is exact in the fp32
// accumulator, and H[i, j] = 2 sum_t sum_{p, q} P_p[t, i] P_q[t, j] differs from
// the CUDA-core kernel's only in the order of its binary32 additions.
namespace ghs {
constexpr int TB = 128;                    // H tile: 128 x 128 (MMA M = N = 128)
constexpr int TS = 64;                     // tokens per stage (one 128-byte swizzled row of bf16)
constexpr int PIECE_BYTES = TB * TS * 2;   // 16 KiB: one piece of one operand
constexpr int STAGE_BYTES = 6 * PIECE_BYTES;   // A pieces 0-2, B pieces 0-2
constexpr int STAGES = 2;
constexpr int THREADS = 256;               // warp 0 loads, warp 1 issues, warp 2 allocates, warps 4-7 store
constexpr int TMEM_COLS = 256;             // two accumulators of 128 columns
constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + 1024 + 256;
constexpr int XT_TILE = 32;                // transpose tile of the prep kernel
}  // namespace ghs

// xt[p][k][t] (bf16, t padded to Tp with zeros): piece p of x'[t, k], k-major
// rows for the tensor-core Hessian, through a 32 x 32 shared-memory transpose.
__global__ void __launch_bounds__(256) gptq_hprep_kernel(const __half *__restrict__ X, int64_t T, int64_t K,
                                                         int64_t ldx, int64_t Tp, const float *__restrict__ s,
                                                         __nv_bfloat16 *__restrict__ xt) {
    using namespace ghs;
    __shared__ __nv_bfloat16 tile[3][XT_TILE][XT_TILE + 2];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;     // 8 rows of 32 a pass
    const int64_t k0 = (int64_t)blockIdx.x * XT_TILE, t0 = (int64_t)blockIdx.y * XT_TILE;
    for (int r = ty; r < XT_TILE; r += 8) {
        const int64_t t = t0 + r, k = k0 + tx;
        float hi = 0.0f, mid = 0.0f, lo = 0.0f;
        if (t < T && k < K) {
            const float xp = __fmul_rn(__half2float(X[t * ldx + k]), __frcp_rn(s[k]));
            hi = __bfloat162float(__float2bfloat16_rn(xp));
            const float r1 = __fsub_rn(xp, hi);                    // exact
            mid = __bfloat162float(__float2bfloat16_rn(r1));
            lo = __fsub_rn(r1, mid);                               // exact, at most 8 bits
        }
        tile[0][r][tx] = __float2bfloat16_rn(hi);
        tile[1][r][tx] = __float2bfloat16_rn(mid);
        tile[2][r][tx] = __float2bfloat16_rn(lo);
    }
    __syncthreads();
    for (int r = ty; r < XT_TILE; r += 8) {
        const int64_t k = k0 + r, t = t0 + tx;
        if (k < K && t < Tp) {
#pragma unroll
            for (int p = 0; p < 3; ++p) xt[((int64_t)p * K + k) * Tp + t] = tile[p][tx][r];
        }
    }
}

// Persistent over the 128 x 128 tiles (bi >= bj) of H's lower block triangle.
// Warp 0 loads, per stage of 64 tokens, the three pieces of rows bi (A) and bj
// (B) with TMA; warp 1 issues the 9 piece pairs x 4 MMAs of K 16 into the tile's
// accumulator (two in tensor memory, so one tile's stores overlap the next
// tile's MMAs); warps 4-7 read the accumulator, one row of the tile per thread,
// and store 2 D to H[i, j] and its mirror H[j, i] (the diagonal tile from its
// lower half only), so H is exactly symmetric.
__global__ void __launch_bounds__(ghs::THREADS, 1)
gptq_hessian_tc_kernel(const __grid_constant__ CUtensorMap tmap_xt, int64_t K, int64_t n_ts, float *__restrict__ H,
                       uint64_t timeout_ns) {
    using namespace ghs;
    constexpr uint32_t IDESC = mma_idesc_bf16_f32(TB, TB);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + STAGES * STAGE_BYTES);
    uint64_t *full = bars, *empty = bars + STAGES, *d_full = bars + 2 * STAGES, *d_empty = d_full + 2;
    uint64_t *drain = d_empty + 2;
    __shared__ uint32_t tmem_base_sm;
    __shared__ int abort_sm;
    volatile int *abort_flag = &abort_sm;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = (int)((K + TB - 1) / TB);
    const int n_tiles = nb * (nb + 1) / 2;
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&d_full[i], 1); mbar_init(&d_empty[i], 4); }
        mbar_init(drain, 1);
        abort_sm = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc_1(&tmem_base_sm, TMEM_COLS);
        tmem_relinquish_1();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sm;
    bool aborted = false;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmap_xt);
            int st = 0;
            uint32_t ph = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !aborted; tile += gridDim.x) {
                int bi, bj;
                lower_block(tile, bi, bj);
                for (int64_t ts = 0; ts < n_ts; ++ts) {
                    if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, timeout_ns)) { aborted = true; break; }
                    mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
                    uint8_t *sb = base + st * STAGE_BYTES;
#pragma unroll
                    for (int p = 0; p < 3; ++p) {
                        tma_load_2d(sb + p * PIECE_BYTES, &tmap_xt, (int32_t)(ts * TS), (int32_t)(p * K + bi * TB),
                                    &full[st]);
                        tma_load_2d(sb + (3 + p) * PIECE_BYTES, &tmap_xt, (int32_t)(ts * TS),
                                    (int32_t)(p * K + bj * TB), &full[st]);
                    }
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int st = 0, db = 0;
            uint32_t ph = 0, dph = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !aborted; tile += gridDim.x) {
                if (!mbar_wait_bounded(&d_empty[db], dph ^ 1u, abort_flag, timeout_ns)) { aborted = true; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(db * TB);
                for (int64_t ts = 0; ts < n_ts; ++ts) {
                    if (!mbar_wait_bounded(&full[st], ph, abort_flag, timeout_ns)) { aborted = true; break; }
                    tc_fence_after();
                    const uint64_t d0 = sw128_kmajor_desc(smem_u32(base + st * STAGE_BYTES));
#pragma unroll
                    for (int p = 0; p < 3; ++p)
#pragma unroll
                        for (int q = 0; q < 3; ++q)
#pragma unroll
                            for (int kk = 0; kk < TS / 16; ++kk)
                                mma_f16_ss_1(d, d0 + (uint64_t)((p * PIECE_BYTES + kk * 32) >> 4),
                                             d0 + (uint64_t)(((3 + q) * PIECE_BYTES + kk * 32) >> 4), IDESC,
                                             (ts | p | q | kk) != 0 ? 1u : 0u);
                    mma_commit_1(&empty[st]);
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
                if (aborted) break;
                mma_commit_1(&d_full[db]);
                if (++db == 2) { db = 0; dph ^= 1u; }
            }
            mma_commit_1(drain);                   // every MMA issued has finished when this fires
            mbar_wait_bounded(drain, 0, abort_flag, timeout_ns);
        }
    } else if (warp >= 4) {
        const int q4 = warp - 4;
        const int rr = 32 * q4 + lane;             // the thread's row of the tile
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        int db = 0;
        uint32_t dph = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            int bi, bj;
            lower_block(tile, bi, bj);
            if (!mbar_wait_warp(&d_full[db], dph, abort_flag, timeout_ns)) { aborted = true; break; }
            tc_fence_after();
            const int64_t i = (int64_t)bi * TB + rr;
            for (int c0 = 0; c0 < TB; c0 += 32) {
                float v[32];
                tmem_ld_32x32b_x32_sync(tmem + lane_base + (uint32_t)(db * TB + c0), v);
                const int64_t j0 = (int64_t)bj * TB + c0;
                // direct: H[i, j] for j <= i on the diagonal tile, all j off it
                if (i < K) {
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        const int64_t j = j0 + c;
                        if (j + 3 < K && (bi != bj || j + 3 <= i)) {
                            *reinterpret_cast<float4 *>(H + i * K + j) =
                                make_float4(2.0f * v[c], 2.0f * v[c + 1], 2.0f * v[c + 2], 2.0f * v[c + 3]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                if (j + e < K && (bi != bj || j + e <= i)) H[i * K + j + e] = 2.0f * v[c + e];
                        }
                    }
                }
                // mirror: H[j, i] for j < i on the diagonal tile, all j off it (coalesced over the warp's rows)
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int64_t j = j0 + c;
                    if (i < K && j < K && (bi != bj || j < i)) H[j * K + i] = 2.0f * v[c];
                }
            }
            tc_fence_before();
            __syncwarp();                          // every lane's reads are complete (wait::ld)
            if (lane == 0) mbar_arrive(&d_empty[db]);
            if (++db == 2) { db = 0; dph ^= 1u; }
        }
    }

    if (aborted || *abort_flag) {                  // let copies in flight land before the block exits
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_1(tmem, TMEM_COLS);
    }
}


// damp * mean(diag H), the damping term: one block, the diagonal summed in
// index order in binary64 (the result does not depend on the launch).
__global__ void __launch_bounds__(256)
gptq_damp_kernel(const float *__restrict__ H, int64_t K, float damp, float *__restrict__ add) {
    __shared__ double part[256];
    double sum = 0.0;
    for (int64_t i = threadIdx.x; i < K; i += 256) sum += (double)H[i * K + i];
    part[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        double tot = 0.0;
        for (int i = 0; i < 256; ++i) tot += part[i];
        *add = __fmul_rn(damp, (float)(tot / (double)K));
    }
}

// A = P (H + add I) P: the damped Hessian with the order of rows and columns
// reversed.
__global__ void gptq_reverse_kernel(const float *__restrict__ H, int64_t K, const float *__restrict__ add,
                                    float *__restrict__ A) {
    const float ad = *add;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < K * K; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / K, j = e - i * K;
        const float v = H[(K - 1 - i) * K + (K - 1 - j)];
        A[e] = i == j ? __fadd_rn(v, ad) : v;
    }
}

// Cholesky, step p of the blocked right-looking form on A (lower, row-major):
// the diagonal block, right-looking inside it.  Thread (r, q) holds row r's
// entries k = q, q + 4, ... in registers.  Column c: the owner of (c, c) takes
// the square root, the owners of (r, c) below divide by it, and every entry
// c < k <= r subtracts L[r][c] L[k][c] (fmaf).  Each entry so receives
// fmaf(-L[r][m], L[k][m], .) for m = 0, 1, ... in order, the sequence of forming
// A[r][k] - sum_m L[r][m] L[k][m] left to right.  A pivot that is not positive
// raises the not-positive-definite flag (and is replaced by 1 so the rest stays
// finite).
constexpr int kCholDiagThreads = 4 * kGb;
__global__ void __launch_bounds__(kCholDiagThreads) chol_diag_kernel(float *__restrict__ A, int64_t K, int p) {
    __shared__ float col[2][kGb];                // column c of L, by parity of c
    const int64_t o = (int64_t)p * kGb;
    const int r = threadIdx.x >> 2, q = threadIdx.x & 3;
    float acc[kGb / 4];
#pragma unroll
    for (int i = 0; i < kGb / 4; ++i) {
        const int k = 4 * i + q;
        acc[i] = k <= r ? A[(o + r) * K + o + k] : 0.0f;
    }
#pragma unroll
    for (int c = 0; c < kGb; ++c) {
        float *cl = col[c & 1];
        if (r == c && q == (c & 3)) {
            float v = acc[c >> 2];
            if (!(v > 0.0f)) { atomicOr(&g_dev_error, kDevErrNotPD); v = 1.0f; }
            acc[c >> 2] = __fsqrt_rn(v);
            cl[c] = acc[c >> 2];
        }
        __syncthreads();
        if (r > c && q == (c & 3)) {
            acc[c >> 2] = __fdiv_rn(acc[c >> 2], cl[c]);
            cl[r] = acc[c >> 2];
        }
        __syncthreads();
        if (r > c) {
            const float lrc = cl[r];
#pragma unroll
            for (int i = 0; i < kGb / 4; ++i) {
                const int k = 4 * i + q;
                if (k > c && k <= r) acc[i] = __fmaf_rn(-lrc, cl[k], acc[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kGb / 4; ++i) {
        const int k = 4 * i + q;
        if (k <= r) A[(o + r) * K + o + k] = acc[i];
    }
}

// Cholesky step p: the panel below the diagonal block, A[i][p] <- A[i][p] L_pp^-T,
// one block row per CTA, one row per thread (forward substitution).
__global__ void __launch_bounds__(kGb) chol_panel_kernel(float *__restrict__ A, int64_t K, int p) {
    __shared__ float L[kGb][kGb + 1];
    const int64_t o = (int64_t)p * kGb;
    const int64_t r0 = o + kGb + (int64_t)blockIdx.x * kGb;
    for (int e = threadIdx.x; e < kGb * kGb; e += kGb) L[e / kGb][e % kGb] = A[(o + e / kGb) * K + o + e % kGb];
    __syncthreads();
    float x[kGb];
    const int64_t row = r0 + threadIdx.x;
#pragma unroll
    for (int c = 0; c < kGb; ++c) x[c] = A[row * K + o + c];
#pragma unroll
    for (int c = 0; c < kGb; ++c) {
        float v = x[c];
#pragma unroll
        for (int m = 0; m < c; ++m) v = __fmaf_rn(-x[m], L[c][m], v);
        x[c] = __fdiv_rn(v, L[c][c]);
    }
#pragma unroll
    for (int c = 0; c < kGb; ++c) A[row * K + o + c] = x[c];
}

// 64 x 64 x 64 block product on shared-memory tiles: acc[a][b] += sum_m P[r][m] Q[c][m]
// for this thread's 4 x 4 patch, rows r = ty*4+a of P and rows c = tx+16b of Q (a
// warp's 16 Q rows then fall in distinct bank groups), m in order; 16-byte loads
// of 4 consecutive m.  Tiles are 16-byte aligned with rows of kGb + 4 floats.
__device__ __forceinline__ int mm_col(int tx, int b) { return tx + 16 * b; }
__device__ __forceinline__ void block_mm_nt(const float (*P)[kGb + 4], const float (*Q)[kGb + 4], int ty, int tx,
                                            float (&acc)[4][4]) {
#pragma unroll 2
    for (int m = 0; m < kGb; m += 4) {
        float4 pv[4], qv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            pv[a] = *reinterpret_cast<const float4 *>(&P[ty * 4 + a][m]);
            qv[a] = *reinterpret_cast<const float4 *>(&Q[mm_col(tx, a)][m]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = __fmaf_rn(pv[a].x, qv[b].x, acc[a][b]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = __fmaf_rn(pv[a].y, qv[b].y, acc[a][b]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = __fmaf_rn(pv[a].z, qv[b].z, acc[a][b]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = __fmaf_rn(pv[a].w, qv[b].w, acc[a][b]);
    }
}

// Cholesky step p: trailing update A[i][j] -= L[i][p] L[j][p]^T for the lower
// blocks p < j <= i, one block per CTA.
__global__ void __launch_bounds__(256) chol_update_kernel(float *__restrict__ A, int64_t K, int p) {
    __shared__ __align__(16) float Pi[kGb][kGb + 4];
    __shared__ __align__(16) float Pj[kGb][kGb + 4];
    int bi, bj;
    lower_block(blockIdx.x, bi, bj);
    bi += p + 1;
    bj += p + 1;
    const int64_t o = (int64_t)p * kGb, i0 = (int64_t)bi * kGb, j0 = (int64_t)bj * kGb;
    for (int e = threadIdx.x; e < kGb * kGb; e += 256) {
        Pi[e / kGb][e % kGb] = A[(i0 + e / kGb) * K + o + e % kGb];
        Pj[e / kGb][e % kGb] = A[(j0 + e / kGb) * K + o + e % kGb];
    }
    __syncthreads();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
    block_mm_nt(Pi, Pj, ty, tx, acc);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float *d = &A[(i0 + ty * 4 + a) * K + j0 + mm_col(tx, b)];
            *d = __fsub_rn(*d, acc[a][b]);
        }
}

// Inverse of the lower factor, M = L^-1, diagonal blocks: thread c solves
// L_pp x = e_c by forward substitution.
__global__ void __launch_bounds__(kGb) trinv_diag_kernel(const float *__restrict__ L, int64_t K,
                                                         float *__restrict__ M) {
    __shared__ float Lp[kGb][kGb + 1];
    const int64_t o = (int64_t)blockIdx.x * kGb;
    for (int e = threadIdx.x; e < kGb * kGb; e += kGb) Lp[e / kGb][e % kGb] = L[(o + e / kGb) * K + o + e % kGb];
    __syncthreads();
    const int c = threadIdx.x;
    float x[kGb];
#pragma unroll
    for (int r = 0; r < kGb; ++r) {
        float v = r == c ? 1.0f : 0.0f;
#pragma unroll
        for (int m = 0; m < r; ++m) v = __fmaf_rn(-Lp[r][m], x[m], v);
        x[r] = r < c ? 0.0f : __fdiv_rn(v, Lp[r][r]);
    }
#pragma unroll
    for (int r = 0; r < kGb; ++r) M[(o + r) * K + o + c] = x[r];
}

// Off-diagonal blocks, right-looking: U's strictly lower blocks first hold
// the pending sums S[i][j] = sum_{k=j}^{i-1} L[i][k] M[k][j], built one block
// column k at a time (fmaf in k order, then m order within a tile), and
// become M[i][j] = -M[i][i] S[i][j] when block row i is final.
// Round k, step 1: block row k's off-diagonal blocks become final.
__global__ void __launch_bounds__(256) trinv_final_kernel(int64_t K, int k, float *__restrict__ M) {
    __shared__ __align__(16) float Pa[kGb][kGb + 4];
    __shared__ __align__(16) float Qb[kGb][kGb + 4];
    const int bj = blockIdx.x;
    const int64_t i0 = (int64_t)k * kGb, j0 = (int64_t)bj * kGb;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    for (int e = threadIdx.x; e < kGb * kGb; e += 256) {
        Pa[e / kGb][e % kGb] = M[(i0 + e / kGb) * K + i0 + e % kGb];        // M[k][k]
        Qb[e % kGb][e / kGb] = M[(i0 + e / kGb) * K + j0 + e % kGb];        // S[k][j], transposed
    }
    __syncthreads();
    float out[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) out[a][b] = 0.0f;
    block_mm_nt(Pa, Qb, ty, tx, out);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) M[(i0 + ty * 4 + a) * K + j0 + mm_col(tx, b)] = -out[a][b];
}

// Round k, step 2: S[i][j] += L[i][k] M[k][j] for every block row i > k and
// block column j <= k, one block per CTA.
__global__ void __launch_bounds__(256) trinv_update_kernel(const float *__restrict__ L, int64_t K, int k,
                                                           float *__restrict__ M) {
    __shared__ __align__(16) float Pa[kGb][kGb + 4];
    __shared__ __align__(16) float Qb[kGb][kGb + 4];
    const int bi = k + 1 + blockIdx.x / (k + 1), bj = blockIdx.x % (k + 1);
    const int64_t i0 = (int64_t)bi * kGb, j0 = (int64_t)bj * kGb, k0 = (int64_t)k * kGb;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    for (int e = threadIdx.x; e < kGb * kGb; e += 256) {
        Pa[e / kGb][e % kGb] = L[(i0 + e / kGb) * K + k0 + e % kGb];        // L[i][k]
        Qb[e % kGb][e / kGb] = M[(k0 + e / kGb) * K + j0 + e % kGb];        // M[k][j], transposed
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = M[(i0 + ty * 4 + a) * K + j0 + mm_col(tx, b)];
    block_mm_nt(Pa, Qb, ty, tx, acc);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) M[(i0 + ty * 4 + a) * K + j0 + mm_col(tx, b)] = acc[a][b];
}

// U = P M P restricted to the upper triangle, in place: element (a, b) and
// (K-1-a, K-1-b) trade places; everything below the diagonal becomes 0.
__global__ void gptq_rotate_kernel(float *__restrict__ M, int64_t K) {
    const int64_t half = (K * K + 1) / 2;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < half; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t a = e / K, b = e - a * K, e2 = K * K - 1 - e;
        const float v1 = M[e], v2 = M[e2];
        // after the swap M[e] holds the old M[e2]; (a, b) is upper iff b >= a
        M[e] = b >= a ? v2 : 0.0f;
        const int64_t a2 = e2 / K, b2 = e2 - a2 * K;
        if (e2 != e) M[e2] = b2 >= a2 ? v1 : 0.0f;
    }
}

// Output error of a given W_hat through the search kernel: dW = RN16(W_hat - W)
// is written as the "weights", and every group's parameters are those of a
// quantizer whose clamp range is the single code z = 0 (qmax = 0, clamp flag
// set), so the kernel's W_hat is 0 and it contracts -dW against X.
__global__ void weight_diff_kernel(const __half *__restrict__ W, const __half *__restrict__ W_hat, int64_t total,
                                   __half *__restrict__ dW) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
        dW[i] = __float2half_rn(__fsub_rn(__half2float(W_hat[i]), __half2float(W[i])));
}
__global__ void zero_code_params_kernel(uint2 *__restrict__ params, int64_t total) {
    QParams p;
    p.r = 1.0f;
    p.sh = 1.0f;
    p.z = 0.0f;
    p.clamp = true;
    const uint2 v = pack_qparams(p);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
        params[i] = v;
}
__global__ void fill_kernel(float *__restrict__ x, int64_t total, float v) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
        x[i] = v;
}

// The GPTQ column sweep over R rows of W per block, binary32, bit for bit the
// sequence of the definition:
//   w = RN32(W s); for k = 0 .. K-1:
//     at a group's first column: the group's parameters from its current w
//     q  = clamp(rint(w_k r) + z, 0, qmax)         (one FMA with 1.5 2^23)
//     wq = RN32((q - z) sh);  e = RN32(RN32(w_k - wq) / U_kk)
//     w_j = fmaf(-e, U_kj, w_j), j > k
// in batches of B consecutive columns (B divides the group size).  The 256
// worker threads own column pairs (pair p goes to thread p mod 256) of all R
// rows and keep those weights in registers.  Per batch: the owners of the
// batch's pairs (and, at a group's start, of the group's pairs) publish those
// weights to shared memory; row warp r settles the batch's B columns of row r
// one after another (each taking the updates of the batch's earlier columns,
// in order) and publishes its B errors; then every owner applies the B
// updates to each of its later weights in column order -- the same fmaf
// sequence per element as one column at a time.  Each pair of U is read once
// per block and used for all R rows.  Warp 8 streams the batch's B rows of U
// into a ring of slots, RING - 1 batches ahead.  Codes go to shared memory and
// are packed at the end;
// W_hat = RN16(RN32(wq RN32(1/s))) is written as each column settles.
namespace gsw {
constexpr int WARPS = 8;                 // worker warps; the first R are also the row warps
constexpr int OWNERS = WARPS * 32;       // worker threads: thread t owns column pairs t + OWNERS i
constexpr int THREADS = WARPS * 32;      // two warps per scheduler: up to 255 registers a thread
constexpr int ISSUER = OWNERS - 1;       // the worker thread that also issues the copies of U rows
constexpr int MAX_RING = 8;
struct Args {
    const __half *W;
    int64_t N, K;
    const float *s, *U;
    int group, G, bits, sym;
    int ring;                            // slots of B rows of U, 2..MAX_RING
    float qmax;
    uint32_t *codes;
    __half *scales, *zeros, *W_hat;
    uint64_t timeout_ns;
};
// shared memory: ring [ring][B][K] floats, published group weights [R][128],
// errors [R][B], codes [R][K] bytes, barriers
inline size_t smem_bytes(int64_t K, int R, int B, int ring) {
    return (size_t)ring * B * K * 4 + (size_t)R * 128 * 4 + (size_t)R * B * 4 + (size_t)R * K + MAX_RING * 8 + 512;
}
}  // namespace gsw

template <int SLOTS, int R, int B>   // pairs per thread (K <= 2 OWNERS SLOTS), rows per block, columns per batch
__global__ void __launch_bounds__(gsw::THREADS, 1) gptq_sweep_kernel(const gsw::Args A) {
    using namespace gsw;
    extern __shared__ uint8_t smem_raw[];
    const int64_t K = A.K;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int RING = A.ring;
    float *ring = reinterpret_cast<float *>(base);                         // [RING][B][K]
    float *pub = ring + (size_t)RING * B * K;                              // [R][128]: weights of a group / a batch
    float *err = pub + R * 128;                                            // [R][B]
    uint8_t *qrow = reinterpret_cast<uint8_t *>(err + R * B);              // [R][K]
    uint64_t *full = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(qrow + (size_t)R * K) + 7) & ~uintptr_t(7));
    __shared__ int abort_flag;
    __shared__ int stop;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int64_t row0 = (int64_t)blockIdx.x * R;
    const int active = (int)(A.N - row0 < R ? A.N - row0 : R);
    const int64_t nbatch = K / B;
    // batch bi's B rows of U into slot bi % RING, from the 16-byte boundary at or
    // below its first column k0 = B bi (a bulk copy needs it; K % 4 == 0)
    auto issue = [&](int64_t bi) {
        const int64_t k0 = bi * B, c0 = k0 & ~int64_t(3);
        const int s = (int)(bi % RING);
        const uint32_t bytes = (uint32_t)((K - c0) * 4);
        mbar_arrive_expect_tx(&full[s], B * bytes);
#pragma unroll
        for (int m = 0; m < B; ++m)
            bulk_load(ring + ((size_t)s * B + m) * K + c0, A.U + (k0 + m) * K + c0, bytes, &full[s]);
    };
    if (tid == 0) {
        for (int i = 0; i < RING; ++i) mbar_init(&full[i], 1);
        abort_flag = 0;
        stop = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == ISSUER)                           // the first RING - 1 batches
        for (int64_t b = 0; b < RING - 1 && b < nbatch; ++b) issue(b);

    // this thread's weights (workers only): pair p = tid + OWNERS i, rows 0..R-1
    float2 wr[SLOTS][R];
    if (warp < WARPS) {
#pragma unroll
        for (int i = 0; i < SLOTS; ++i) {
            const int64_t p = tid + OWNERS * (int64_t)i;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float2 v = make_float2(0.0f, 0.0f);
                if (2 * p < K && r < active) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(A.W + (row0 + r) * K + 2 * p));
                    v = make_float2(__fmul_rn(f.x, A.s[2 * p]), __fmul_rn(f.y, A.s[2 * p + 1]));
                }
                wr[i][r] = v;
            }
        }
    }
    QParams prm{};                               // row warp `warp`'s current group parameters
    for (int64_t bi = 0; bi < nbatch; ++bi) {
        const int64_t k0 = bi * B;
        const int sl = (int)(bi % RING);
        const uint32_t par = (uint32_t)((bi / RING) & 1);
        const bool gstart = k0 % A.group == 0;
        const int npub = gstart ? A.group : B;
        // (a) owners publish the group's weights at its start, else the batch's
        if (warp < WARPS) {
#pragma unroll
            for (int i = 0; i < SLOTS; ++i) {
                const int64_t p = tid + OWNERS * (int64_t)i;
                if (2 * p >= k0 && 2 * p < k0 + npub) {
#pragma unroll
                    for (int r = 0; r < R; ++r) *reinterpret_cast<float2 *>(pub + r * 128 + (2 * p - k0)) = wr[i][r];
                }
            }
        }
        __syncthreads();                         // every worker is past batch bi-1: its slot is free
        if (tid == ISSUER && bi + RING - 1 < nbatch) issue(bi + RING - 1);
        // (b) row warp r settles the batch's columns of row r; every worker waits for the slot.
        // Lane i < B reads s of column k0 + i first, so the load is off the column chain.
        const float s_lane = (warp < active && lane < B) ? __ldg(A.s + k0 + lane) : 1.0f;
        bool ok = true;
        if (warp < WARPS) ok = mbar_wait_warp(&full[sl], par, &abort_flag, A.timeout_ns);
        if (ok && warp < active) {
            const int r = warp;
            const float *pw = pub + r * 128;
            if (gstart) {
                float mn = INFINITY, mx = -INFINITY;
                for (int j = lane; j < A.group; j += 32) { mn = fminf(mn, pw[j]); mx = fmaxf(mx, pw[j]); }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                }
                prm = make_qparams(mn, mx, A.qmax, A.sym != 0);
                if (lane == 0) {
                    A.scales[(row0 + r) * A.G + k0 / A.group] = __float2half_rn(prm.sh);
                    A.zeros[(row0 + r) * A.G + k0 / A.group] = __float2half_rn(prm.z);
                }
            }
            const float *Ub = ring + (size_t)sl * B * K;
            const float vlo = __fsub_rn(kMagic, prm.z), vhi = __fadd_rn(kMagic, __fsub_rn(A.qmax, prm.z));
            float e[B];
            float q_l = 0.0f, wq_l = 0.0f, e_l = 0.0f;   // lane i keeps column k0 + i's results
#pragma unroll
            for (int i = 0; i < B; ++i) {
                float wk = pw[i];
#pragma unroll
                for (int m = 0; m < i; ++m) wk = __fmaf_rn(-e[m], Ub[m * K + k0 + i], wk);
                const float v = fminf(fmaxf(__fmaf_rn(wk, prm.r, kMagic), vlo), vhi);
                const float qf = __fsub_rn(v, vlo);
                const float wq = __fmul_rn(__fsub_rn(qf, prm.z), prm.sh);
                e[i] = __fdiv_rn(__fsub_rn(wk, wq), Ub[i * K + k0 + i]);
                if (lane == i) {
                    q_l = qf;
                    wq_l = wq;
                    e_l = e[i];
                }
            }
            if (lane < B) {
                qrow[(size_t)r * K + k0 + lane] = (uint8_t)q_l;
                A.W_hat[(row0 + r) * K + k0 + lane] = __float2half_rn(__fmul_rn(wq_l, __frcp_rn(s_lane)));
                err[r * B + lane] = e_l;
            }
        }
        if (!ok && lane == 0) atomicExch(&stop, 1);
        __syncthreads();
        if (stop) break;
        // (c) every owner: the B updates of each later weight, in column order
        if (warp < WARPS) {
            const float *Ub = ring + (size_t)sl * B * K;
            float ne[R][B];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < B; ++m) ne[r][m] = r < active ? -err[r * B + m] : 0.0f;
            const int64_t pstart = (k0 + B) / 2;
#pragma unroll
            for (int i = 0; i < SLOTS; ++i) {
                const int64_t p = tid + OWNERS * (int64_t)i;
                if (p >= pstart && 2 * p < K) {
                    float2 u[B];
#pragma unroll
                    for (int m = 0; m < B; ++m) u[m] = *reinterpret_cast<const float2 *>(Ub + m * K + 2 * p);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        float2 v = wr[i][r];
#pragma unroll
                        for (int m = 0; m < B; ++m) v = fma2_rn(make_float2(ne[r][m], ne[r][m]), u[m], v);
                        wr[i][r] = v;
                    }
                }
            }
        }
    }
    __syncthreads();
    // codes (least-significant first)
    if (!stop && warp < WARPS) {
        const int c = A.bits == 2 ? 2 : 4, per = 32 / c;
        const int64_t words = K / per;
        for (int64_t e = tid; e < (int64_t)active * words; e += WARPS * 32) {
            const int r = (int)(e / words);
            const int64_t wd = e - (int64_t)r * words;
            uint32_t v = 0;
            for (int i = 0; i < per; ++i) v |= (uint32_t)qrow[(size_t)r * K + wd * per + i] << (c * i);
            A.codes[(row0 + r) * words + wd] = v;
        }
    }
    // copies still in flight (an abort) land before the block leaves
    if (abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    __syncthreads();
}

// ===========================================================================
// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// ever arrives on.  The wait gives up after the library's limit, raises the
// device timeout flag and returns -- the path every role of the search kernel
// takes when a pipeline stalls.  (Library infrastructure; the pages have no
// counterpart.)
// ===========================================================================
__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, timeout_ns);
    __syncthreads();
}

}  // namespace awq
