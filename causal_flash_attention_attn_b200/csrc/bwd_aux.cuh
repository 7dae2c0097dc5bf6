// bwd_aux.cuh -- the two HBM-bound stages around the backward main kernel.
//  preprocess: Delta_i = sum_d dO_id * o_id (f32), the row term of the softmax
//              gradient dS_ij = P_ij (dP_ij - Delta_i); one warp per row.
//  finalize:   dq = bf16(dq accumulator) for the tensor-core path.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"

namespace forge {

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
__device__ __forceinline__ void load8(const float *p, float (&f)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// rows = B*Hq*T; D a multiple of 8 (64/128/256). A row takes LPR = min(32, D/8)
// lanes, each loading 8-element chunks d = 8*(sub + LPR*i), so a warp covers
// 32/LPR rows at once and every lane loads (head dim 64: four rows a warp).
// When `acc` is given, the matching row of the dq accumulator ([BH][Tpad][D]
// f32) is zeroed too (rows past T are never read).
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_preprocess(const T *__restrict__ o, const T *__restrict__ dO,
                                                      float *__restrict__ delta, float *__restrict__ acc, long rows,
                                                      int T_, int Tpad) {
    constexpr int LPR = D / 8 < 32 ? D / 8 : 32;  // lanes per row
    constexpr int RPW = 32 / LPR;                  // rows per warp
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x % 32, sub = lane % LPR;
    const long row = ((long)blockIdx.x * 8 + threadIdx.x / 32) * RPW + lane / LPR;
    const bool live = row < rows;
    const long r = live ? row : rows - 1;  // every lane takes part in the shuffles below
    if (acc != nullptr && live) {
        float *arow = acc + ((r / T_) * Tpad + r % T_) * D;
        for (int c = sub * 4; c < D; c += 4 * LPR) *reinterpret_cast<float4 *>(arow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const T *orow = o + r * D;
    const T *drow = dO + r * D;
    float sum = 0.0f;
    for (int c = sub * 8; c < D; c += 8 * LPR) {
        float a[8], b[8];
        load8(orow + c, a);
        load8(drow + c, b);
#pragma unroll
        for (int i = 0; i < 8; i++) sum = fmaf(a[i], b[i], sum);
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (sub == 0 && live) delta[r] = sum;
}

// dq[bh][t][:] = bf16(acc[bh][t][:]) for t < T; acc rows are padded to Tpad.
template <int D>
__global__ void __launch_bounds__(256) bwd_finalize_dq(const float *__restrict__ acc, __nv_bfloat16 *__restrict__ dq,
                                                       long BH, int T_, int Tpad) {
    constexpr int CH = D / 8;  // 8-element chunks per row
    griddep_launch_dependents();
    griddep_wait();
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const long total = BH * T_ * CH;
    if (idx >= total) return;
    const int c = idx % CH;
    const long row = idx / CH;
    const long bh = row / T_;
    const int t = row % T_;
    float f[8];
    load8(acc + ((bh * Tpad + t) * D + c * 8), f);
    uint4 u;
    uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(dq + (row * D + c * 8)) = u;
}

}  // namespace forge
