// simt.cuh -- CUDA-core attention kernels (f32 arithmetic throughout).
//
// This is the f32 path of the library (FORGE_DTYPE_F32): exact f32 FMAs, no
// tensor cores, so the result stays within the 1e-4 parity bar the Forge pages
// set for their CPU-vs-GPU checks (the Forge README: every parity check within 1e-4).
//
// Structure: a block owns 16 rows (4 warps x 4 rows); keys (or queries) stream
// through shared memory 32 at a time; lane j of a warp scores element j of the
// tile, and lane d owns output columns d, d+32, ...
//  - simt_fwd:   rows = queries; online softmax over key tiles -> o, lse.
//  - simt_bwd_dq: rows = queries; P = exp(s - lse), dS = P (dP - Delta) [* cap'],
//                 dq = scale * sum dS k.
//  - simt_bwd_dkdv: rows = keys; loops over the group's query heads and the
//                 queries that see the key; dv = sum P dO, dk = scale * sum dS q.
// No atomics: every output element has one writer, so results are deterministic.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "sm100.cuh"

namespace forge {

constexpr int kSimtRows = 16;  // rows per block
constexpr int kSimtTile = 32;  // streamed rows per tile
constexpr int kSimtThreads = 128;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f32(float *p, float x) { *p = x; }
__device__ __forceinline__ void from_f32(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Index of the (batch, head) pair a block works on. Launches put the pairs on
// grid y and, past the 65535 that y allows, on z (host side: `pair_grid`); the
// blocks of the last z slice beyond the pair count return before any work.
__device__ __forceinline__ int pair_index() { return (int)(blockIdx.y + gridDim.y * blockIdx.z); }

// Visible iff kj <= qi and (window == 0 or kj > qi - window).
__device__ __forceinline__ bool visible(int qi, int kj, int window) {
    return kj <= qi && (window == 0 || kj > qi - window);
}

// Capped score from the scaled dot product (natural units).
__device__ __forceinline__ float simt_capped(float s, float softcap) {
    return softcap > 0.0f ? softcap * tanhf(s / softcap) : s;
}

template <typename T, int D>
__device__ __forceinline__ void load_rows(float *dst, int ld, const T *src, int row0, int nrows,
                                          int T_) {
    for (int idx = threadIdx.x; idx < nrows * D; idx += blockDim.x) {
        const int r = idx / D, d = idx % D;
        dst[r * ld + d] = (row0 + r < T_ && row0 + r >= 0) ? to_f32(src[(size_t)(row0 + r) * D + d]) : 0.0f;
    }
}

// DK: head dim of q and k; DV: head dim of v and o (equal except for the
// decompressed multi-head latent attention, d_k = 192, d_v = 128).
template <int DK, int DV>
constexpr size_t simt_fwd_smem() {
    return sizeof(float) * (size_t)(kSimtRows * DK + kSimtTile * (DK + 1) + kSimtTile * (DV + 1));
}

// Minimum resident CTAs a kernel asks ptxas to allow for: as many as its shared
// memory admits on one SM (228 KB, 1 KB of it reserved per CTA), at most eight.
// The register cap this implies never costs occupancy that shared memory does not
// already cost, and it leaves ptxas room to keep the accumulators out of local memory.
constexpr int simt_min_blocks(size_t smem) {
    return (int)(233472 / (smem + 1024)) < 8 ? (int)(233472 / (smem + 1024)) : 8;
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads, simt_min_blocks(simt_fwd_smem<DK, DV>()))
    simt_fwd(const T *__restrict__ q, const T *__restrict__ k,
             const T *__restrict__ v, T *__restrict__ o,
             float *__restrict__ lse, int Hq, int Hkv, int T_,
             float scale, int window, float softcap,
             const float *__restrict__ sink, float *__restrict__ max_logit, int npairs) {
    extern __shared__ float sm[];
    float *sQ = sm;
    float *sK = sQ + kSimtRows * DK;
    float *sV = sK + kSimtTile * (DK + 1);
    constexpr int NT = DV / 32;
    const int bh = pair_index(), b = bh / Hq, hq = bh % Hq, hkv = hq / (Hq / Hkv);
    if (bh >= npairs) return;
    const int r0 = blockIdx.x * kSimtRows;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const T *Qb = q + (size_t)bh * T_ * DK;
    const T *Kb = k + (size_t)(b * Hkv + hkv) * T_ * DK;
    const T *Vb = v + (size_t)(b * Hkv + hkv) * T_ * DV;
    load_rows<T, DK>(sQ, DK, Qb, r0, kSimtRows, T_);

    // a sink (natural units) starts each row's (max, sum) at (sink, 1)
    float m[4], l[4], acc[4][NT], mraw[4];
#pragma unroll
    for (int rr = 0; rr < 4; rr++) {
        m[rr] = sink ? sink[hq] : -INFINITY;
        l[rr] = sink ? 1.0f : 0.0f;
        mraw[rr] = -INFINITY;
#pragma unroll
        for (int t = 0; t < NT; t++) acc[rr][t] = 0.0f;
    }
    const int last = min(r0 + kSimtRows - 1, T_ - 1);
    int first = (window > 0) ? max(0, r0 - window + 1) : 0;
    first = (first / kSimtTile) * kSimtTile;
    for (int k0 = first; k0 <= last; k0 += kSimtTile) {
        __syncthreads();
        load_rows<T, DK>(sK, DK + 1, Kb, k0, kSimtTile, T_);
        load_rows<T, DV>(sV, DV + 1, Vb, k0, kSimtTile, T_);
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < 4; rr++) {
            const int r = warp * 4 + rr, qi = r0 + r;
            if (qi >= T_) continue;
            const int kj = k0 + lane;
            float s = 0.0f;
#pragma unroll 8
            for (int d = 0; d < DK; d++) s = fmaf(sQ[r * DK + d], sK[lane * (DK + 1) + d], s);
            s = simt_capped(s * scale, softcap);
            const bool ok = visible(qi, kj, window) && kj < T_;
            s = ok ? s : -INFINITY;
            const float smax = warp_max(s);
            mraw[rr] = fmaxf(mraw[rr], smax);
            const float mnew = fmaxf(m[rr], smax);
            if (mnew == -INFINITY) continue;
            const float corr = expf(m[rr] - mnew);
            const float p = ok ? expf(s - mnew) : 0.0f;
            l[rr] = l[rr] * corr + warp_sum(p);
#pragma unroll
            for (int t = 0; t < NT; t++) acc[rr][t] *= corr;
            for (int j = 0; j < kSimtTile; j++) {
                const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
                for (int t = 0; t < NT; t++) acc[rr][t] = fmaf(pj, sV[j * (DV + 1) + lane + 32 * t], acc[rr][t]);
            }
            m[rr] = mnew;
        }
    }
#pragma unroll
    for (int rr = 0; rr < 4; rr++) {
        const int qi = r0 + warp * 4 + rr;
        if (qi >= T_) continue;
        const float inv = 1.0f / l[rr];
        T *orow = o + ((size_t)bh * T_ + qi) * DV;
#pragma unroll
        for (int t = 0; t < NT; t++) from_f32(orow + lane + 32 * t, acc[rr][t] * inv);
        if (lane == 0) lse[(size_t)bh * T_ + qi] = m[rr] + logf(l[rr]);
        if (max_logit != nullptr && lane == 0) atomic_max_f32(max_logit + bh, mraw[rr]);
    }
}

template <int DK, int DV>
constexpr size_t simt_bwd_dq_smem() {
    return sizeof(float) * (size_t)(kSimtRows * (DK + DV) + kSimtTile * (DK + 1) + kSimtTile * (DV + 1));
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads, simt_min_blocks(simt_bwd_dq_smem<DK, DV>()))
    simt_bwd_dq(const T *__restrict__ q, const T *__restrict__ k,
                const T *__restrict__ v, const float *__restrict__ lse,
                const T *__restrict__ dO, const float *__restrict__ delta,
                T *__restrict__ dq, int Hq, int Hkv, int T_, float scale,
                int window, float softcap, int npairs) {
    extern __shared__ float sm[];
    float *sQ = sm;
    float *sdO = sQ + kSimtRows * DK;
    float *sK = sdO + kSimtRows * DV;
    float *sV = sK + kSimtTile * (DK + 1);
    constexpr int NT = DK / 32;
    const int bh = pair_index(), b = bh / Hq, hq = bh % Hq, hkv = hq / (Hq / Hkv);
    if (bh >= npairs) return;
    const int r0 = blockIdx.x * kSimtRows;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const T *Kb = k + (size_t)(b * Hkv + hkv) * T_ * DK;
    const T *Vb = v + (size_t)(b * Hkv + hkv) * T_ * DV;
    load_rows<T, DK>(sQ, DK, q + (size_t)bh * T_ * DK, r0, kSimtRows, T_);
    load_rows<T, DV>(sdO, DV, dO + (size_t)bh * T_ * DV, r0, kSimtRows, T_);
    float acc[4][NT], L[4], Dl[4];
#pragma unroll
    for (int rr = 0; rr < 4; rr++) {
        const int qi = min(r0 + warp * 4 + rr, T_ - 1);
        L[rr] = lse[(size_t)bh * T_ + qi];
        Dl[rr] = delta[(size_t)bh * T_ + qi];
#pragma unroll
        for (int t = 0; t < NT; t++) acc[rr][t] = 0.0f;
    }
    const int last = min(r0 + kSimtRows - 1, T_ - 1);
    int first = (window > 0) ? max(0, r0 - window + 1) : 0;
    first = (first / kSimtTile) * kSimtTile;
    for (int k0 = first; k0 <= last; k0 += kSimtTile) {
        __syncthreads();
        load_rows<T, DK>(sK, DK + 1, Kb, k0, kSimtTile, T_);
        load_rows<T, DV>(sV, DV + 1, Vb, k0, kSimtTile, T_);
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < 4; rr++) {
            const int r = warp * 4 + rr, qi = r0 + r;
            if (qi >= T_) continue;
            const int kj = k0 + lane;
            float s = 0.0f, dp = 0.0f;
#pragma unroll 8
            for (int d = 0; d < DK; d++) s = fmaf(sQ[r * DK + d], sK[lane * (DK + 1) + d], s);
#pragma unroll 8
            for (int d = 0; d < DV; d++) dp = fmaf(sdO[r * DV + d], sV[lane * (DV + 1) + d], dp);
            const float sc = simt_capped(s * scale, softcap);
            const bool ok = visible(qi, kj, window) && kj < T_;
            const float p = ok ? expf(sc - L[rr]) : 0.0f;
            float ds = p * (dp - Dl[rr]);
            if (softcap > 0.0f) {
                const float t = sc / softcap;
                ds *= 1.0f - t * t;
            }
            for (int j = 0; j < kSimtTile; j++) {
                const float dsj = __shfl_sync(0xffffffffu, ds, j);
#pragma unroll
                for (int t = 0; t < NT; t++) acc[rr][t] = fmaf(dsj, sK[j * (DK + 1) + lane + 32 * t], acc[rr][t]);
            }
        }
    }
#pragma unroll
    for (int rr = 0; rr < 4; rr++) {
        const int qi = r0 + warp * 4 + rr;
        if (qi >= T_) continue;
        T *row = dq + ((size_t)bh * T_ + qi) * DK;
#pragma unroll
        for (int t = 0; t < NT; t++) from_f32(row + lane + 32 * t, acc[rr][t] * scale);
    }
}

template <int DK, int DV>
constexpr size_t simt_bwd_dkdv_smem() {
    return sizeof(float) *
           (size_t)(kSimtRows * (DK + DV) + kSimtTile * (DK + 1) + kSimtTile * (DV + 1) + 2 * kSimtTile);
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads, simt_min_blocks(simt_bwd_dkdv_smem<DK, DV>()))
    simt_bwd_dkdv(const T *__restrict__ q, const T *__restrict__ k,
                  const T *__restrict__ v, const float *__restrict__ lse,
                  const T *__restrict__ dO,
                  const float *__restrict__ delta, T *__restrict__ dk,
                  T *__restrict__ dv, int Hq, int Hkv, int T_,
                  float scale, int window, float softcap, int npairs) {
    extern __shared__ float sm[];
    float *sK = sm;                          // [16][DK] key rows of this block
    float *sV = sK + kSimtRows * DK;         // [16][DV]
    float *sQ = sV + kSimtRows * DV;         // [32][DK+1] query tile
    float *sdO = sQ + kSimtTile * (DK + 1);  // [32][DV+1]
    float *sL = sdO + kSimtTile * (DV + 1);  // [32]
    float *sD = sL + kSimtTile;              // [32]
    constexpr int NK = DK / 32, NV = DV / 32;
    const int bkv = pair_index(), b = bkv / Hkv, hkv = bkv % Hkv;
    if (bkv >= npairs) return;
    const int G = Hq / Hkv;
    const int r0 = blockIdx.x * kSimtRows;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    load_rows<T, DK>(sK, DK, k + (size_t)bkv * T_ * DK, r0, kSimtRows, T_);
    load_rows<T, DV>(sV, DV, v + (size_t)bkv * T_ * DV, r0, kSimtRows, T_);
    float adk[4][NK], adv[4][NV];
#pragma unroll
    for (int rr = 0; rr < 4; rr++) {
#pragma unroll
        for (int t = 0; t < NK; t++) adk[rr][t] = 0.0f;
#pragma unroll
        for (int t = 0; t < NV; t++) adv[rr][t] = 0.0f;
    }
    const int qfirst = (r0 / kSimtTile) * kSimtTile;
    int qlast = T_ - 1;
    if (window > 0) qlast = min(qlast, r0 + kSimtRows - 1 + window - 1);
    for (int g = 0; g < G; g++) {
        const int bh = b * Hq + hkv * G + g;
        for (int q0 = qfirst; q0 <= qlast; q0 += kSimtTile) {
            __syncthreads();
            load_rows<T, DK>(sQ, DK + 1, q + (size_t)bh * T_ * DK, q0, kSimtTile, T_);
            load_rows<T, DV>(sdO, DV + 1, dO + (size_t)bh * T_ * DV, q0, kSimtTile, T_);
            if (threadIdx.x < kSimtTile) {
                const int qi = q0 + threadIdx.x;
                sL[threadIdx.x] = qi < T_ ? lse[(size_t)bh * T_ + qi] : 0.0f;
                sD[threadIdx.x] = qi < T_ ? delta[(size_t)bh * T_ + qi] : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int rr = 0; rr < 4; rr++) {
                const int r = warp * 4 + rr, kj = r0 + r;
                if (kj >= T_) continue;
                const int qi = q0 + lane;
                float s = 0.0f, dp = 0.0f;
#pragma unroll 8
                for (int d = 0; d < DK; d++) s = fmaf(sK[r * DK + d], sQ[lane * (DK + 1) + d], s);
#pragma unroll 8
                for (int d = 0; d < DV; d++) dp = fmaf(sV[r * DV + d], sdO[lane * (DV + 1) + d], dp);
                const float sc = simt_capped(s * scale, softcap);
                const bool ok = qi < T_ && visible(qi, kj, window);
                const float p = ok ? expf(sc - sL[lane]) : 0.0f;
                float ds = p * (dp - sD[lane]);
                if (softcap > 0.0f) {
                    const float t = sc / softcap;
                    ds *= 1.0f - t * t;
                }
                for (int j = 0; j < kSimtTile; j++) {
                    const float pj = __shfl_sync(0xffffffffu, p, j);
                    const float dsj = __shfl_sync(0xffffffffu, ds, j);
#pragma unroll
                    for (int t = 0; t < NV; t++) adv[rr][t] = fmaf(pj, sdO[j * (DV + 1) + lane + 32 * t], adv[rr][t]);
#pragma unroll
                    for (int t = 0; t < NK; t++) adk[rr][t] = fmaf(dsj, sQ[j * (DK + 1) + lane + 32 * t], adk[rr][t]);
                }
            }
        }
    }
#pragma unroll
    for (int rr = 0; rr < 4; rr++) {
        const int kj = r0 + warp * 4 + rr;
        if (kj >= T_) continue;
        T *krow = dk + ((size_t)bkv * T_ + kj) * DK;
        T *vrow = dv + ((size_t)bkv * T_ + kj) * DV;
#pragma unroll
        for (int t = 0; t < NK; t++) from_f32(krow + lane + 32 * t, adk[rr][t] * scale);
#pragma unroll
        for (int t = 0; t < NV; t++) from_f32(vrow + lane + 32 * t, adv[rr][t]);
    }
}

}  // namespace forge
