// decode.cuh -- one-query attention against a KV cache, split over the keys.
//
// INFERENCE_RESEARCH.md section 2 (KV cache): the cache is pre-allocated to the
// maximum length with a layout coalesced along time per head ([layer][head][seq][d];
// one layer's [B][Hkv][Tmax][D] here), and decoding gets a dedicated kernel: one
// query, split-K along the cache for long contexts; GQA is the largest saving of
// KV bandwidth. The work is HBM-bound (each cache byte is read once and feeds
// 2*G flops per element), so it runs on the CUDA cores with pipelined
// asynchronous loads rather than on the tensor cores.
//
// Two split kernels share the (key chunk, batch entry, KV head) decomposition:
// decode_split_warp (below; every warp an independent pipeline) where the
// group's queries fit a lane's registers, decode_split otherwise.
//
// decode_split: one CTA per (key chunk, batch entry, KV head), all G query heads
// of the group at once, so every K/V byte is read once for the G heads. K/V
// tiles of KT keys stream through a STAGES-deep cp.async ring (rows past the
// chunk end are zero-filled); per tile: scores in log2 units (the query is
// pre-scaled, or the cap applied), an online softmax per head, then P.V. The
// chunk's unnormalised (max, sum, o) per head go to the workspace.
// decode_combine: one CTA per (batch entry, query head) merges the chunks and the
// optional sink, writes o and lse.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "bwd_aux.cuh"
#include "simt.cuh"
#include "sm100.cuh"

namespace forge {

constexpr int kDecThreads = 256;
constexpr int kDecMaxG = 16;  // query heads per KV head supported by the decode kernels

template <typename T_, int D>
struct DecCfg {
    static constexpr int ROWB = D * (int)sizeof(T_);            // bytes of one cache row
    static constexpr int KT = ROWB <= 512 ? 64 : 32;            // keys per tile
    static constexpr int PITCH = ROWB + 16;                     // padded smem row: rows land on other banks
    static constexpr int TILEB = KT * PITCH;                    // one K or V tile in smem
    static constexpr int PIECES = KT * ROWB / 16;               // 16-byte pieces of a tile
    static constexpr int STAGES = 2;  // two tiles in flight per CTA; several CTAs per SM
    // scores: thread -> (key pair tid / SQ, slice tid % SQ of SL head dims), all
    // heads; the query slices are padded so that the SQ slices of a warp's loads
    // fall on different banks
    static constexpr int SQ = kDecThreads / (KT / 2);           // 8 (KT 64) or 16 (KT 32)
    static constexpr int SL = D / SQ;                           // head dims per slice
    static constexpr int QP = SL + 4;                           // padded slice length (floats)
    // P.V: thread -> (head-dim pair tid % (D / 2), key group tid / (D / 2)), all
    // heads; the key groups' sums are added once, after the last tile
    static constexpr int NKG = kDecThreads / (D / 2);           // key groups: 8, 4, 2 for D 64, 128, 256
    static constexpr int KG = KT / NKG;                         // keys of a group per tile
    // shared memory for G query heads: q [G][SQ][QP], p [G][KT] f32, (max, sum,
    // correction) per head, then the K/V tile ring (16-byte aligned), which the
    // final key-group reduction [NKG][G][D] f32 reuses
    static constexpr size_t f32_words(int G) { return (size_t)G * SQ * QP + (size_t)G * KT + 3 * (size_t)G; }
    static constexpr size_t tiles_off(int G) { return (f32_words(G) * 4 + 15) / 16 * 16; }
    static constexpr size_t smem(int G) { return tiles_off(G) + (size_t)STAGES * 2 * TILEB; }
    static_assert(smem(kDecMaxG) <= 232448, "shared memory");
    static_assert((size_t)NKG * kDecMaxG * D * 4 <= (size_t)STAGES * 2 * TILEB, "reduction space");
    static_assert(D % 8 == 0 && kDecThreads % (D / 2) == 0 && KT % 32 == 0 && KG % 4 == 0, "shape");
    static_assert(SL % 8 == 0 && (SQ & (SQ - 1)) == 0 && SQ <= 32, "score slices");
};

struct DecParams {
    const int *seq_lens;  // [B] valid cache lengths, or nullptr (all T)
    const float *sink;    // [Hq] or nullptr
    float *part;          // [B*Hq][nsplit][D + 2]: max (log2 units), sum, o[D] (unnormalised)
    float *lse;           // [B*Hq] or nullptr
    int B, Hq, Hkv, T, Tmax, window, chunk, nsplit;
    float qscale;         // scale * log2(e) without a cap, scale / softcap with one
    float cap_out;        // softcap * log2(e), 0 without a cap
};

__device__ __forceinline__ void load2(const float *p, float (&f)[2]) {
    const float2 v = *reinterpret_cast<const float2 *>(p);
    f[0] = v.x;
    f[1] = v.y;
}
__device__ __forceinline__ void load2(const __nv_bfloat16 *p, float (&f)[2]) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
    f[0] = v.x;
    f[1] = v.y;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// MG: the smallest of 4, 8, 16 that holds the group's G query heads (sizes the
// per-thread accumulators)
template <typename T_, int D, int MG>
__global__ void __launch_bounds__(kDecThreads) decode_split(const T_ *__restrict__ q, const T_ *__restrict__ kc,
                                                            const T_ *__restrict__ vc, const DecParams p) {
    using C = DecCfg<T_, D>;
    extern __shared__ __align__(16) uint8_t dsm[];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int bkv = pair_index(), b = bkv / p.Hkv, hkv = bkv % p.Hkv, split = blockIdx.x;
    if (bkv >= p.B * p.Hkv) return;
    const int G = p.Hq / p.Hkv;
    float *q_s = reinterpret_cast<float *>(dsm);  // [G][SQ][QP], pre-scaled
    float *p_s = q_s + G * C::SQ * C::QP;         // [G][KT] scores, then probabilities
    float *m_s = p_s + G * C::KT;                 // [G] running max (log2 units)
    float *l_s = m_s + G;                         // [G] running sum
    float *c_s = l_s + G;                         // [G] this tile's correction factor
    uint8_t *tiles = dsm + C::tiles_off(G);
    const uint32_t tiles_s = smem_u32(tiles);

    int len = p.seq_lens ? p.seq_lens[b] : p.T;
    if (len < 1 || len > p.T) {
        // a length outside [1, T] would leave keys unread: report it, process nothing
        if (tid == 0) record_status(kStatusInvalidArg);
        len = 0;
    }
    const int lo = p.window > 0 ? max(0, len - p.window) : 0;
    const int c0 = max(lo, split * p.chunk), c1 = min(len, (split + 1) * p.chunk);
    const size_t hstride = (size_t)p.nsplit * (D + 2);
    float *part = p.part + ((size_t)(b * p.Hq + hkv * G) * p.nsplit + split) * (D + 2);
    if (c0 >= c1) {
        for (int idx = tid; idx < G * (D + 2); idx += kDecThreads) {
            const int g = idx / (D + 2), e = idx % (D + 2);
            part[g * hstride + e] = e == 0 ? -INFINITY : 0.0f;
        }
        return;
    }

    const T_ *Kb = kc + (size_t)bkv * p.Tmax * D;
    const T_ *Vb = vc + (size_t)bkv * p.Tmax * D;
    const int ntiles = (c1 - c0 + C::KT - 1) / C::KT;
    auto load_tile = [&](int t) {
        if (t < ntiles) {
            const int k0 = c0 + t * C::KT;
            const uint32_t kt = tiles_s + (uint32_t)((t % C::STAGES) * 2 * C::TILEB), vt = kt + C::TILEB;
            for (int c = tid; c < C::PIECES; c += kDecThreads) {
                const int r = c / (C::ROWB / 16), w = c % (C::ROWB / 16);
                const int key = k0 + r;
                const bool in = key < c1;
                const size_t goff = (size_t)(in ? key : c0) * C::ROWB + (size_t)w * 16;  // valid even when unread
                const uint32_t soff = (uint32_t)(r * C::PITCH + w * 16);
                cp_async16(kt + soff, reinterpret_cast<const uint8_t *>(Kb) + goff, in ? 16 : 0);
                cp_async16(vt + soff, reinterpret_cast<const uint8_t *>(Vb) + goff, in ? 16 : 0);
            }
        }
        cp_async_commit();  // an empty group past the end keeps the wait counts uniform
    };
    for (int t = 0; t < C::STAGES - 1; t++) load_tile(t);

    // the G queries, f32, pre-scaled, in padded slices; running (max, sum) per head
    for (int idx = tid; idx < G * D; idx += kDecThreads) {
        const int g = idx / D, d = idx % D;
        q_s[(g * C::SQ + d / C::SL) * C::QP + d % C::SL] =
            to_f32(q[(size_t)(b * p.Hq + hkv * G) * D + idx]) * p.qscale;
    }
    if (tid < G) {
        m_s[tid] = -INFINITY;
        l_s[tid] = 0.0f;
    }
    const int sk = tid / C::SQ, sl = tid % C::SQ;        // scores: key pair, slice
    const int pd2 = tid % (D / 2), kg = tid / (D / 2);   // P.V: head-dim pair, key group
    float acc[MG][2];
#pragma unroll
    for (int g = 0; g < MG; g++) acc[g][0] = acc[g][1] = 0.0f;

    for (int t = 0; t < ntiles; t++) {
        cp_async_wait<C::STAGES - 2>();
        __syncthreads();  // tile t landed for every thread; tile t - 1 fully consumed
        load_tile(t + C::STAGES - 1);
        const uint8_t *kt = tiles + (size_t)(t % C::STAGES) * 2 * C::TILEB, *vt = kt + C::TILEB;
        const int nk = min(C::KT, c1 - (c0 + t * C::KT));
        // scores of keys 2 sk, 2 sk + 1 over slice sl, every head; the SQ slices
        // of a key pair are adjacent lanes and add their parts by shuffles
        {
            const int j0 = 2 * sk;
            float k0[C::SL], k1[C::SL];
            const T_ *r0 = reinterpret_cast<const T_ *>(kt + j0 * C::PITCH) + sl * C::SL;
            const T_ *r1 = reinterpret_cast<const T_ *>(kt + (j0 + 1) * C::PITCH) + sl * C::SL;
#pragma unroll
            for (int d = 0; d < C::SL; d += 8) {
                float f[8];
                load8(r0 + d, f);
#pragma unroll
                for (int e = 0; e < 8; e++) k0[d + e] = f[e];
                load8(r1 + d, f);
#pragma unroll
                for (int e = 0; e < 8; e++) k1[d + e] = f[e];
            }
            // all heads' dot products first (independent chains), then their
            // slice reductions interleaved
            float a0[MG], a1[MG];
#pragma unroll
            for (int g = 0; g < MG; g++) {
                a0[g] = a1[g] = 0.0f;
                if (g < G) {
                    const float4 *qg = reinterpret_cast<const float4 *>(q_s + (g * C::SQ + sl) * C::QP);
#pragma unroll
                    for (int d4 = 0; d4 < C::SL / 4; d4++) {
                        const float4 qv = qg[d4];
                        a0[g] = fmaf(qv.x, k0[4 * d4], a0[g]);
                        a1[g] = fmaf(qv.x, k1[4 * d4], a1[g]);
                        a0[g] = fmaf(qv.y, k0[4 * d4 + 1], a0[g]);
                        a1[g] = fmaf(qv.y, k1[4 * d4 + 1], a1[g]);
                        a0[g] = fmaf(qv.z, k0[4 * d4 + 2], a0[g]);
                        a1[g] = fmaf(qv.z, k1[4 * d4 + 2], a1[g]);
                        a0[g] = fmaf(qv.w, k0[4 * d4 + 3], a0[g]);
                        a1[g] = fmaf(qv.w, k1[4 * d4 + 3], a1[g]);
                    }
                }
            }
#pragma unroll
            for (int o = C::SQ / 2; o > 0; o >>= 1) {
#pragma unroll
                for (int g = 0; g < MG; g++) {
                    if (g < G) {
                        a0[g] += __shfl_xor_sync(0xffffffffu, a0[g], o);
                        a1[g] += __shfl_xor_sync(0xffffffffu, a1[g], o);
                    }
                }
            }
            if (sl == 0) {
#pragma unroll
                for (int g = 0; g < MG; g++) {
                    if (g < G) {
                        float s0 = a0[g], s1 = a1[g];
                        if (p.cap_out > 0.0f) {
                            s0 = p.cap_out * tanhf(s0);
                            s1 = p.cap_out * tanhf(s1);
                        }
                        p_s[g * C::KT + j0] = j0 < nk ? s0 : -INFINITY;
                        p_s[g * C::KT + j0 + 1] = j0 + 1 < nk ? s1 : -INFINITY;
                    }
                }
            }
        }
        __syncthreads();
        // online softmax per head: warp w takes heads w, w + 8, ...
        for (int g = warp; g < G; g += kDecThreads / 32) {
            float sv[C::KT / 32];
            float mx = -INFINITY;
#pragma unroll
            for (int u = 0; u < C::KT / 32; u++) {
                sv[u] = p_s[g * C::KT + lane + 32 * u];
                mx = fmaxf(mx, sv[u]);
            }
            mx = warp_max_f32(mx);
            const float m_old = m_s[g], m_new = fmaxf(m_old, mx);  // finite: the tile has a key
            float sum = 0.0f;
#pragma unroll
            for (int u = 0; u < C::KT / 32; u++) {
                const float e = exp2f(sv[u] - m_new);
                p_s[g * C::KT + lane + 32 * u] = e;
                sum += e;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) {
                const float corr = exp2f(m_old - m_new);
                m_s[g] = m_new;
                l_s[g] = l_s[g] * corr + sum;
                c_s[g] = corr;
            }
        }
        __syncthreads();
        // P.V over this thread's key group, every head (keys past nk: V rows are
        // zero-filled and their probabilities 0)
#pragma unroll
        for (int g = 0; g < MG; g++) {
            if (g < G) {
                const float cr = c_s[g];
                acc[g][0] *= cr;
                acc[g][1] *= cr;
            }
        }
#pragma unroll 1
        for (int j = kg * C::KG; j < (kg + 1) * C::KG; j += 4) {
            float v[4][2];
#pragma unroll
            for (int u = 0; u < 4; u++) load2(reinterpret_cast<const T_ *>(vt + (j + u) * C::PITCH) + 2 * pd2, v[u]);
#pragma unroll
            for (int g = 0; g < MG; g++) {
                if (g < G) {
                    const float4 pv = *reinterpret_cast<const float4 *>(p_s + g * C::KT + j);
                    acc[g][0] = fmaf(pv.x, v[0][0], fmaf(pv.y, v[1][0], fmaf(pv.z, v[2][0], fmaf(pv.w, v[3][0], acc[g][0]))));
                    acc[g][1] = fmaf(pv.x, v[0][1], fmaf(pv.y, v[1][1], fmaf(pv.z, v[2][1], fmaf(pv.w, v[3][1], acc[g][1]))));
                }
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    // add the key groups' sums (in the now idle tile ring), write the partials
    float *red = reinterpret_cast<float *>(tiles);  // [NKG][G][D]
#pragma unroll
    for (int g = 0; g < MG; g++) {
        if (g < G) {
            red[((size_t)kg * G + g) * D + 2 * pd2] = acc[g][0];
            red[((size_t)kg * G + g) * D + 2 * pd2 + 1] = acc[g][1];
        }
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kDecThreads) {
        const int g = idx / D, d = idx % D;
        float sum = 0.0f;
#pragma unroll
        for (int k = 0; k < C::NKG; k++) sum += red[((size_t)k * G + g) * D + d];
        part[g * hstride + 2 + d] = sum;
    }
    if (tid < G) {
        part[tid * hstride + 0] = m_s[tid];
        part[tid * hstride + 1] = l_s[tid];
    }
}

// ---------------------------------------------------------------------------
// decode_split_warp: the same (key chunk, batch entry, KV head) work per CTA,
// with every warp an independent pipeline over its share of the chunk (steps
// w, w + NW, w + 2 NW, ... of KW keys), for groups with MG * D <= 1024 and rows
// of at most 256 * MG bytes. Per warp: its own ring of NST stages filled by
// bulk copies (one for the step's K rows, one for its V rows, completing on the
// stage's mbarrier), the G queries in registers (lane L holds head dims
// L*DL .. L*DL + DL - 1 of every head), its own running max, sum and output.
// Per step, each lane forms partial dot products over its DL dims for the
// KW * MG = 32 (key, head) slots; a transposed shuffle reduction (at each level a
// lane keeps one half of its slots and adds its partner's copy of that half)
// leaves lane L with the full score of slot L (key L / MG, head L % MG), so the
// softmax of the step needs one score per lane and the per-head maximum only
// log2(KW) shuffles. The running max moves only when a step's maximum exceeds
// it by more than 8 (log2 units), so most steps skip the rescale of o. P.V: each
// lane accumulates its DL dims of every head from the V rows and the step's
// probabilities (through shared memory, read as broadcasts). No CTA barrier
// runs until the warps merge their (max, sum, o) at the end.
constexpr int kDecWarps = 4;
constexpr int kDecWRing = 8192;  // bytes of K/V ring per warp (about)

template <typename T_, int D, int MG>
struct DecWCfg {
    static constexpr int DL = D / 32;                  // head dims per lane
    static constexpr int KW = 32 / MG;                 // keys per step: 32 (key, head) slots
    static constexpr int ROWB = D * (int)sizeof(T_);   // bytes of one cache row
    static constexpr int SEGB = DL * (int)sizeof(T_);  // bytes of a lane's part of a row
    static constexpr int STEPB = KW * ROWB;            // K (or V) bytes of one step
    static constexpr int STAGEB = 2 * STEPB;
    static constexpr int NST = kDecWRing / STAGEB < 2 ? 2 : (kDecWRing / STAGEB > 8 ? 8 : kDecWRing / STAGEB);
    static constexpr int RING = kDecWarps * NST * STAGEB;
    // after the ring: mbarriers [NW][NST], p [NW][32] as (p, p) pairs,
    // correction [NW][MG], max and sum [NW][MG] each, the abort flag
    static constexpr int OFF_BAR = RING;
    static constexpr int OFF_P = OFF_BAR + kDecWarps * NST * 8;
    static constexpr int OFF_C = OFF_P + kDecWarps * 32 * 8;
    static constexpr int OFF_M = OFF_C + kDecWarps * MG * 4;
    static constexpr int OFF_L = OFF_M + kDecWarps * MG * 4;
    static constexpr int OFF_ABORT = OFF_L + kDecWarps * MG * 4;
    static constexpr int SMEM = OFF_ABORT + 16;
    static_assert(MG * D <= 1024 && STEPB <= 8192, "shape served by decode_split");
    static_assert((size_t)kDecWarps * MG * D * 4 <= (size_t)RING, "merge space");
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(ROWB % 16 == 0 && SEGB % 4 == 0 && (MG & (MG - 1)) == 0 && DL % 2 == 0, "shape");
};

// A lane's DL elements of a row as DL / 2 packed f32 pairs (element 2i in the
// low half): bf16 -> f32 is a 16-bit shift (low element) or a mask (high one).
template <typename T_, int DL>
__device__ __forceinline__ void load_seg2(const uint8_t *p, uint64_t (&f)[DL / 2]) {
    if constexpr (sizeof(T_) == 2) {
        uint32_t w[DL / 2];
        if constexpr (DL == 2) {
            w[0] = *reinterpret_cast<const uint32_t *>(p);
        } else if constexpr (DL == 4) {
            const uint2 u = *reinterpret_cast<const uint2 *>(p);
            w[0] = u.x; w[1] = u.y;
        } else {
            const uint4 u = *reinterpret_cast<const uint4 *>(p);
            w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
        }
#pragma unroll
        for (int i = 0; i < DL / 2; i++) f[i] = f2_make(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
    } else {
#pragma unroll
        for (int i = 0; i < DL / 2; i++) f[i] = *reinterpret_cast<const uint64_t *>(p + 8 * i);
    }
}

// v[r] (32 partial sums per lane) -> the warp-wide sum of slot `lane`. Slot
// e = key * MG + head; register r of lane L holds slot r ^ (L & ~(MG - 1)) (the
// caller reads key rows in that lane-permuted order), so at the levels that
// reduce over key bits (offsets 16 .. MG) every lane keeps its lower half of
// registers and sends the upper half, with no per-lane selection; the levels
// over head bits (offsets MG / 2 .. 1) pick the half by the lane's bit.
template <int MG>
__device__ __forceinline__ float warp_transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o >= MG; o >>= 1) {
#pragma unroll
        for (int i = 0; i < o; i++) v[i] += __shfl_xor_sync(0xffffffffu, v[i + o], o);
    }
#pragma unroll
    for (int o = MG / 2; o > 0; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; i++) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

template <typename T_, int D, int MG>
__global__ void __launch_bounds__(kDecWarps * 32) decode_split_warp(const T_ *__restrict__ q,
                                                                    const T_ *__restrict__ kc,
                                                                    const T_ *__restrict__ vc, const DecParams p) {
    using C = DecWCfg<T_, D, MG>;
    extern __shared__ __align__(16) uint8_t dsm[];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int bkv = pair_index(), b = bkv / p.Hkv, hkv = bkv % p.Hkv, split = blockIdx.x;
    if (bkv >= p.B * p.Hkv) return;
    const int G = p.Hq / p.Hkv;
    const uint32_t ring = smem_u32(dsm) + (uint32_t)(warp * C::NST * C::STAGEB);
    const uint32_t bars = smem_u32(dsm + C::OFF_BAR) + (uint32_t)(warp * C::NST * 8);
    float *pw = reinterpret_cast<float *>(dsm + C::OFF_P) + warp * 64;  // (p, p) per slot
    float *cw = reinterpret_cast<float *>(dsm + C::OFF_C) + warp * MG;
    float *m_s = reinterpret_cast<float *>(dsm + C::OFF_M);
    float *l_s = reinterpret_cast<float *>(dsm + C::OFF_L);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(dsm + C::OFF_ABORT);

    int len = p.seq_lens ? p.seq_lens[b] : p.T;
    if (len < 1 || len > p.T) {
        if (tid == 0) record_status(kStatusInvalidArg);
        len = 0;
    }
    const int lo = p.window > 0 ? max(0, len - p.window) : 0;
    const int c0 = max(lo, split * p.chunk), c1 = min(len, (split + 1) * p.chunk);
    const size_t hstride = (size_t)p.nsplit * (D + 2);
    float *part = p.part + ((size_t)(b * p.Hq + hkv * G) * p.nsplit + split) * (D + 2);
    if (c0 >= c1) {
        for (int idx = tid; idx < G * (D + 2); idx += kDecWarps * 32) {
            const int g = idx / (D + 2), e = idx % (D + 2);
            part[g * hstride + e] = e == 0 ? -INFINITY : 0.0f;
        }
        return;
    }
    const uint8_t *Kb = reinterpret_cast<const uint8_t *>(kc + (size_t)bkv * p.Tmax * D);
    const uint8_t *Vb = reinterpret_cast<const uint8_t *>(vc + (size_t)bkv * p.Tmax * D);
    const int nsteps = (c1 - c0 + C::KW - 1) / C::KW;
    // this warp's steps: w + j * NW for j = 0, 1, ...
    const int nj = warp < nsteps ? (nsteps - warp + kDecWarps - 1) / kDecWarps : 0;
    auto issue = [&](int j) {  // lane 0: step j of this warp into stage j % NST
        const int k0 = c0 + (warp + j * kDecWarps) * C::KW;
        const uint32_t bytes = (uint32_t)(min(C::KW, c1 - k0) * C::ROWB);
        const uint32_t st = ring + (uint32_t)((j % C::NST) * C::STAGEB), bar = bars + (uint32_t)((j % C::NST) * 8);
        mbar_arrive_expect_tx(bar, 2 * bytes);
        bulk_load(st, Kb + (size_t)k0 * C::ROWB, bytes, bar);
        bulk_load(st + C::STEPB, Vb + (size_t)k0 * C::ROWB, bytes, bar);
    };
    if (tid == 0) *abort_flag = 0;
    if (lane == 0) {
        for (int s = 0; s < C::NST; s++) mbar_init(bars + 8 * s, 1);
        fence_mbar_init();
    }
    __syncthreads();  // the abort flag and every warp's barriers are initialised
    if (lane == 0) {
        for (int j = 0; j < C::NST && j < nj; j++) issue(j);
    }
    // the queries of the group (pre-scaled), this lane's head dims
    // (packed f32 pairs of consecutive head dims)
    uint64_t q2[MG][C::DL / 2], acc2[MG][C::DL / 2];
#pragma unroll
    for (int g = 0; g < MG; g++) {
#pragma unroll
        for (int i = 0; i < C::DL / 2; i++) {
            const T_ *qg = q + (size_t)(b * p.Hq + hkv * G + g) * D + lane * C::DL + 2 * i;
            q2[g][i] = g < G ? f2_make(to_f32(qg[0]) * p.qscale, to_f32(qg[1]) * p.qscale) : f2_make(0.0f, 0.0f);
            acc2[g][i] = f2_make(0.0f, 0.0f);
        }
    }
    // this lane's slot: key lane / MG of a step, head lane % MG
    const int key_l = lane / MG, g_l = lane % MG;
    float m_run = -INFINITY, l_run = 0.0f;  // the slot's head: running max (log2 units), this lane's sum
    bool ok = true;
    int j = 0;
    for (; j < nj; j++) {
        const uint32_t st = ring + (uint32_t)((j % C::NST) * C::STAGEB);
        if (!(ok = mbar_wait_warp(bars + (uint32_t)((j % C::NST) * 8), (uint32_t)((j / C::NST) & 1), abort_flag)))
            break;
        const int k0 = c0 + (warp + j * kDecWarps) * C::KW;
        const int nk = min(C::KW, c1 - k0);
        const uint8_t *kt = dsm + (st - smem_u32(dsm)), *vt = kt + C::STEPB;
        // partial scores over this lane's dims: register k * MG + g takes key row
        // k ^ key_l (the order warp_transpose_sum32 expects). Rows past nk hold
        // stale data; their slots are masked below.
        float sc[32];
#pragma unroll
        for (int k = 0; k < C::KW; k++) {
            uint64_t k2[C::DL / 2];
            load_seg2<T_, C::DL>(kt + (k ^ key_l) * C::ROWB + lane * C::SEGB, k2);
#pragma unroll
            for (int g = 0; g < MG; g++) {
                uint64_t a2 = f2_mul(q2[g][0], k2[0]);
#pragma unroll
                for (int i = 1; i < C::DL / 2; i++) a2 = f2_fma(q2[g][i], k2[i], a2);
                float x, y;
                f2_split(a2, x, y);
                sc[k * MG + g] = x + y;
            }
        }
        float s = warp_transpose_sum32<MG>(sc, lane);
        if (p.cap_out > 0.0f) s = p.cap_out * tanhf(s);
        s = key_l < nk ? s : -INFINITY;
        float mx = s;
#pragma unroll
        for (int o = MG; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_new = mx > m_run + 8.0f ? mx : m_run;  // finite: the step has a key
        const float corr = exp2f(m_run - m_new);
        const float pr = exp2f(s - m_new);
        l_run = fmaf(l_run, corr, pr);
        const bool rescale = __any_sync(0xffffffffu, m_new != m_run);
        m_run = m_new;
        *reinterpret_cast<float2 *>(pw + 2 * lane) = make_float2(pr, pr);
        if (rescale && lane < MG) cw[lane] = corr;
        __syncwarp();
        if (rescale) {
#pragma unroll
            for (int g = 0; g < MG; g++) {
                const float cg = cw[g];
                const uint64_t c2 = f2_make(cg, cg);
#pragma unroll
                for (int i = 0; i < C::DL / 2; i++) acc2[g][i] = f2_mul(acc2[g][i], c2);
            }
        }
#pragma unroll
        for (int k = 0; k < C::KW; k++) {
            if (k < nk) {
                uint64_t v2[C::DL / 2];
                load_seg2<T_, C::DL>(vt + k * C::ROWB + lane * C::SEGB, v2);
                // (p, p) of every head for key k (slots k * MG ..)
                uint64_t p2[MG];
                if constexpr (MG >= 2) {
#pragma unroll
                    for (int g = 0; g < MG; g += 2) {
                        const uint4 t = *reinterpret_cast<const uint4 *>(pw + 2 * (k * MG + g));
                        p2[g] = (uint64_t)t.x | ((uint64_t)t.y << 32);
                        p2[g + 1] = (uint64_t)t.z | ((uint64_t)t.w << 32);
                    }
                } else {
                    p2[0] = *reinterpret_cast<const uint64_t *>(pw + 2 * k);
                }
#pragma unroll
                for (int g = 0; g < MG; g++) {
#pragma unroll
                    for (int i = 0; i < C::DL / 2; i++) acc2[g][i] = f2_fma(p2[g], v2[i], acc2[g][i]);
                }
            }
        }
        __syncwarp();  // every lane is done with the stage and the probabilities
        if (lane == 0 && j + C::NST < nj) {
            fence_proxy_async_smem();
            issue(j + C::NST);
        }
    }
    if (!ok) {
        // let this warp's copies in flight land before the CTA's memory is released
        if (lane == 0) {
            for (int jj = j; jj < nj && jj < j + C::NST; jj++)
                mbar_wait_drain(bars + (uint32_t)((jj % C::NST) * 8), (uint32_t)((jj / C::NST) & 1), 100000000ull);
        }
        __syncwarp();
    }
    // the warp's sum per head (lanes of one head hold parts of it), then the merge
#pragma unroll
    for (int o = MG; o < 32; o <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, o);
    if (key_l == 0) {
        m_s[warp * MG + g_l] = m_run;
        l_s[warp * MG + g_l] = l_run;
    }
    __syncthreads();  // every warp is out of its loop: the ring is free
    float *red = reinterpret_cast<float *>(dsm);  // [NW][MG][D]
#pragma unroll
    for (int g = 0; g < MG; g++) {
#pragma unroll
        for (int i = 0; i < C::DL / 2; i++)
            *reinterpret_cast<uint64_t *>(red + ((size_t)warp * MG + g) * D + lane * C::DL + 2 * i) = acc2[g][i];
    }
    __syncthreads();
    if (*abort_flag) return;
    for (int idx = tid; idx < G * D; idx += kDecWarps * 32) {
        const int g = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; w++) M = fmaxf(M, m_s[w * MG + g]);
        float o = 0.0f, L = 0.0f;
#pragma unroll
        for (int w = 0; w < kDecWarps; w++) {
            const float mw = m_s[w * MG + g];
            if (mw == -INFINITY) continue;  // a warp with no step
            const float f = exp2f(mw - M);
            o = fmaf(red[((size_t)w * MG + g) * D + d], f, o);
            L = fmaf(l_s[w * MG + g], f, L);
        }
        part[g * hstride + 2 + d] = o;
        if (d == 0) {
            part[g * hstride + 0] = M;
            part[g * hstride + 1] = L;
        }
    }
}

// One CTA (D threads) per (batch entry, query head): merge the chunks, then the
// sink: M = max of the chunk maxima (and the sink), L = sum l 2^(m - M), o = sum
// o 2^(m - M) / L, lse = (M + log2 L) ln 2.
template <typename T_, int D>
__global__ void __launch_bounds__(D) decode_combine(T_ *__restrict__ o, const DecParams p) {
    const int bh = blockIdx.x, hq = bh % p.Hq, d = threadIdx.x;
    const float *part = p.part + (size_t)bh * p.nsplit * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < p.nsplit; s++) M = fmaxf(M, part[(size_t)s * (D + 2)]);
    const float sk = p.sink ? p.sink[hq] * kLog2e : -INFINITY;
    const float M2 = fmaxf(M, sk);
    float L = 0.0f, acc = 0.0f;
    for (int s = 0; s < p.nsplit; s++) {
        const float m = part[(size_t)s * (D + 2)];
        if (m == -INFINITY) continue;  // a chunk with no visible key
        const float w = exp2f(m - M2);
        L = fmaf(part[(size_t)s * (D + 2) + 1], w, L);
        acc = fmaf(part[(size_t)s * (D + 2) + 2 + d], w, acc);
    }
    if (p.sink) L += exp2f(sk - M2);
    from_f32(o + (size_t)bh * D + d, acc / L);
    if (p.lse && d == 0) p.lse[bh] = (M2 + log2f(L)) * kLn2;
}

}  // namespace forge
