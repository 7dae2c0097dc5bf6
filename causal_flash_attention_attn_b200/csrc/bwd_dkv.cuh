// bwd_dkv.cuh -- tensor-core backward (bf16 in, f32 accumulate) when the key and
// value head dims differ: the decompressed multi-head latent attention of the
// DeepSeek V3 family, q.k over 192 dims (128 without RoPE + 64 with it), values
// of 128 (ARCHITECTURES.md "Vague 3" item 13; family table, DeepSeek V3 row).
//
// TMEM has 512 columns. One kernel holding S^T, dP^T, dV (DV), dK (DK) and dQ
// does not fit at DK = 192, so the backward runs as two kernels:
//
// bwd_dkdv_tc_kernel -- one CTA per (key tile of 128, batch, KV head), K and V
//   resident in shared memory, dK and dV in TMEM over all G query heads and all
//   query tiles that see the keys (diagonal up to the window's reach). Steps of
//   128 query rows:
//     S^T  = K Q^T  -> columns [0, 128)          P^T (bf16) -> columns PD
//     dP^T = V dO^T -> columns [0, 128) (over S^T, which phase A has read)
//     dV  += P^T dO    (A = P^T from TMEM)
//     dS^T (bf16)   -> columns PD (over P^T, once dV has read it)
//     dK  += dS^T Q    (A = dS^T from TMEM)
//   TMEM: 128 (S^T / dP^T) + DV + DK + 64 (P^T / dS^T) = 512 at (192, 128).
//   Order on the tensor cores: dP^T(i), dV(i), S^T(i + 1), dK(i); dK(i) runs
//   while the compute warps form P of step i + 1, dV(i) while they form dS(i).
//
// bwd_dq_tc_kernel -- one CTA per (query tile of 128 rows, batch, query head),
//   Q and dO resident, dQ in TMEM over the key tiles the rows see (128 keys a
//   tile, K through a two-slot ring since dQ(j) reads K(j) after S(j), V through
//   a one-slot ring, each ring with its own producer warp). The two softmax
//   warpgroups split every tile's keys (64 each) and alternate 128-column TMEM
//   buffers by tile:
//     S  = Q K^T   -> buffer;  P, the dS factor g in registers
//     dP = dO V^T  -> buffer (over S)
//     dS = g (dP - Delta) * scale -> bf16 into the first 32 columns of each half
//     dQ += dS K   (A = dS from TMEM, one K = 64 product per half)
//   Every dQ row is complete in its CTA: no f32 accumulator, no atomics.
//
// Both recompute S and dP: 2 (DK + DV + DV + DK) + 2 (DK + DV + DK) flops per
// allowed pair instead of the 2 (3 DK + 2 DV) of one fused kernel.
#pragma once

#include "bwd_tc.cuh"
#include "fwd_tc.cuh"
#include "sm100.cuh"

namespace forge {

// ------------------------------------------------------------ dK / dV kernel
template <int DK, int DV>
struct BwdKvTc {
    static constexpr int BN = 128, BM = 128;              // keys per CTA, query rows per step
    static constexpr int NCBK = DK / 64, NCBV = DV / 64;  // 64-column (128-byte) blocks
    static constexpr uint32_t CB = 128 * 128;             // one column block of a 128-row tile
    static constexpr uint32_t TK = NCBK * CB;             // K or Q tile
    static constexpr uint32_t TV = NCBV * CB;             // V or dO tile
    static constexpr int QST = 2;                         // Q stages (dO has one)
    static constexpr uint32_t OFF_K = 0, OFF_V = TK, OFF_Q = TK + TV, OFF_DO = OFF_Q + QST * TK;
    static constexpr uint32_t TILES = OFF_DO + TV;
    // control block after the tiles: barriers, TMEM slot, abort flag, per-stage
    // -LSE*log2(e) and -scale*Delta of the step's query rows
    static constexpr uint32_t OFF_TMEM_SLOT = 240, OFF_ABORT = 244, OFF_LSE = 256;
    static constexpr uint32_t OFF_DLT = OFF_LSE + QST * BM * 4;
    static constexpr uint32_t CTRL = OFF_DLT + QST * BM * 4;
    static constexpr uint32_t SMEM = 1024 + TILES + CTRL;  // 1024: alignment of the tiles
    // warps 0-7 compute (warp w: key rows = TMEM lanes 32 (w % 4).., query half
    // w / 4 of the step), warp 8 loads, warp 9 issues MMAs and owns TMEM
    static constexpr int THREADS = 384;
    static constexpr int W_LOAD = 8, W_MMA = 9;
    static constexpr int HALF = BM / 2;
    static constexpr uint32_t COL_S = 0, COL_DV = 128, COL_DK = COL_DV + DV, COL_PD = COL_DK + DK;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_PD + BM / 2 <= TMEM_COLS, "tensor memory");
    static_assert(SMEM <= 232448, "shared memory");
    static constexpr int B_KV = 0, B_Q_FULL = 1, B_Q_EMPTY = 1 + QST, B_DO_FULL = 1 + 2 * QST;
    static constexpr int B_DO_EMPTY = B_DO_FULL + 1, B_S_FULL = B_DO_FULL + 2, B_P_FULL = B_DO_FULL + 3;
    static constexpr int B_DP_FULL = B_DO_FULL + 4, B_DV_DONE = B_DO_FULL + 5, B_DS_FULL = B_DO_FULL + 6;
    static constexpr int B_DK_DONE = B_DO_FULL + 7, B_KDONE = B_DO_FULL + 8;
    static constexpr int NBAR = B_KDONE + 1;
    static_assert(NBAR * 8 <= (int)OFF_TMEM_SLOT, "control block");
};

template <int DK, int DV>
__global__ void __launch_bounds__(384, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const BwdParams p) {
    using C = BwdKvTc<DK, DV>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const uint32_t tiles = (sbase + 1023u) & ~1023u;
    const uint32_t ctrl = tiles + C::TILES;
    uint8_t *const ctrl_p = smem_raw + (ctrl - sbase);
    const uint32_t sK = tiles + C::OFF_K, sV = tiles + C::OFF_V, sQ0 = tiles + C::OFF_Q, sdO = tiles + C::OFF_DO;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl_p + C::OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctrl_p + C::OFF_TMEM_SLOT);
    float *sLSE = reinterpret_cast<float *>(ctrl_p + C::OFF_LSE);
    float *sDLT = reinterpret_cast<float *>(ctrl_p + C::OFF_DLT);
    auto bar = [&](int i) -> uint32_t { return ctrl + 8u * (uint32_t)i; };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // work item: key tile n (heaviest = smallest n first), batch b, KV head
    int n, bkv;
    grouped_block((int)blockIdx.x, p.num_kt, p.B * p.Hkv, n, bkv);
    const int b = bkv / p.Hkv, hkv = bkv % p.Hkv;
    const int G = p.Hq / p.Hkv;
    const int k0 = n * C::BN;
    const int W = p.window;
    const int m_lo = k0 / C::BM;
    const int q_last = W > 0 ? min(p.T - 1, k0 + C::BN - 1 + W - 1) : p.T - 1;
    const int nm = q_last / C::BM - m_lo + 1;
    const int steps = G * nm;

    if (threadIdx.x == 0) {
        mbar_init(bar(C::B_KV), 1);
        for (int s = 0; s < C::QST; s++) {
            mbar_init(bar(C::B_Q_FULL + s), 33);  // expect_tx + the 32 lanes that wrote LSE / Delta
            mbar_init(bar(C::B_Q_EMPTY + s), 1);
        }
        mbar_init(bar(C::B_DO_FULL), 1);
        mbar_init(bar(C::B_DO_EMPTY), 1);
        mbar_init(bar(C::B_S_FULL), 1);
        mbar_init(bar(C::B_P_FULL), 8);
        mbar_init(bar(C::B_DP_FULL), 1);
        mbar_init(bar(C::B_DV_DONE), 1);
        mbar_init(bar(C::B_DS_FULL), 8);
        mbar_init(bar(C::B_DK_DONE), 1);
        mbar_init(bar(C::B_KDONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::W_LOAD && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
    }
    if (warp == C::W_MMA) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::W_LOAD) {
        // ------------------------------------------------------------ producer
        int issued_q = 0, issued_do = 0;
        bool ok = true;
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(C::B_KV), C::TK + C::TV);
            for (int c = 0; c < C::NCBK; c++) tma_load_3d(sK + c * C::CB, &tmK, bar(C::B_KV), c * 64, k0, bkv);
            for (int c = 0; c < C::NCBV; c++) tma_load_3d(sV + c * C::CB, &tmV, bar(C::B_KV), c * 64, k0, bkv);
        }
        for (int i = 0; i < steps; i++) {
            const int st = i % C::QST;
            const int g = i / nm, m = m_lo + i % nm;
            const int bhq = b * p.Hq + hkv * G + g;
            float lv[C::BM / 32], dv[C::BM / 32];
#pragma unroll
            for (int r = 0; r < C::BM / 32; r++) {
                const int q = m * C::BM + lane + 32 * r;
                const size_t idx = (size_t)bhq * p.T + (size_t)min(q, p.T - 1);
                lv[r] = q < p.T ? p.lse[idx] * kLog2e : INFINITY;
                dv[r] = q < p.T ? p.delta[idx] * p.scale : 0.0f;
            }
            if (!mbar_wait_warp(bar(C::B_Q_EMPTY + st), (uint32_t)(((i / C::QST) & 1) ^ 1), abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(C::B_Q_FULL + st), C::TK);
                for (int c = 0; c < C::NCBK; c++)
                    tma_load_3d(sQ0 + st * C::TK + c * C::CB, &tmQ, bar(C::B_Q_FULL + st), c * 64, m * C::BM, bhq);
            }
            issued_q++;
#pragma unroll
            for (int r = 0; r < C::BM / 32; r++) {
                sLSE[st * C::BM + lane + 32 * r] = -lv[r];
                sDLT[st * C::BM + lane + 32 * r] = -dv[r];
            }
            mbar_arrive(bar(C::B_Q_FULL + st));
            if (!mbar_wait_warp(bar(C::B_DO_EMPTY), (uint32_t)((i & 1) ^ 1), abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(C::B_DO_FULL), C::TV);
                for (int c = 0; c < C::NCBV; c++)
                    tma_load_3d(sdO + c * C::CB, &tmdO, bar(C::B_DO_FULL), c * 64, m * C::BM, bhq);
            }
            issued_do++;
        }
        if (!ok && lane == 0) {
            // let the copies already issued land before the CTA exits
            mbar_wait_drain(bar(C::B_KV), 0, 200000000ull);
            for (int back = 1; back <= min(issued_q, C::QST); back++) {
                const int L = issued_q - back;
                mbar_wait_drain(bar(C::B_Q_FULL + L % C::QST), (uint32_t)((L / C::QST) & 1), 200000000ull);
            }
            if (issued_do > 0) mbar_wait_drain(bar(C::B_DO_FULL), (uint32_t)((issued_do - 1) & 1), 200000000ull);
        }
    } else if (warp == C::W_MMA) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_bf16_f32(128, C::BM, false, false);
            constexpr uint32_t ID_DV = idesc_bf16_f32(128, DV, false, true);
            constexpr uint32_t ID_DK = idesc_bf16_f32(128, DK, false, true);
            auto off = [](int kk) -> uint32_t { return (uint32_t)((kk >> 2) * C::CB + (kk & 3) * 32); };
            // S^T(j) = K Q(j)^T over the key head dim
            auto issue_s = [&](int j) -> bool {
                const int st = j % C::QST;
                if (!mbar_wait(bar(C::B_Q_FULL + st), (uint32_t)((j / C::QST) & 1), abort_flag)) return false;
                tc_fence_after();
                const uint32_t sQ = sQ0 + st * C::TK;
#pragma unroll
                for (int kk = 0; kk < DK / 16; kk++)
                    mma_ss(tmem + C::COL_S, sdesc_sw128(sK + off(kk), 16, 1024), sdesc_sw128(sQ + off(kk), 16, 1024),
                           ID_S, kk > 0);
                tc_commit(bar(C::B_S_FULL));
                return true;
            };
            bool ok = mbar_wait(bar(C::B_KV), 0, abort_flag);
            if (ok) ok = issue_s(0);
            for (int i = 0; ok && i < steps; i++) {
                const int st = i % C::QST;
                const uint32_t sQ = sQ0 + st * C::TK;
                // phase A of step i done: S^T(i) read, P^T(i) in TMEM
                if (!(ok = mbar_wait(bar(C::B_P_FULL), (uint32_t)(i & 1), abort_flag))) break;
                if (!(ok = mbar_wait(bar(C::B_DO_FULL), (uint32_t)(i & 1), abort_flag))) break;
                tc_fence_after();
                // dP^T(i) = V dO(i)^T over S^T(i)
#pragma unroll
                for (int kk = 0; kk < DV / 16; kk++)
                    mma_ss(tmem + C::COL_S, sdesc_sw128(sV + off(kk), 16, 1024), sdesc_sw128(sdO + off(kk), 16, 1024),
                           ID_S, kk > 0);
                tc_commit(bar(C::B_DP_FULL));
                // dV += P^T dO (dO MN-major: N = the value head dim)
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; kk++)
                    mma_ts(tmem + C::COL_DV, tmem + C::COL_PD + 8 * kk, sdesc_sw128(sdO + kk * 2048, C::CB, 1024),
                           ID_DV, (i > 0 || kk > 0) ? 1u : 0u);
                tc_commit(bar(C::B_DV_DONE));
                tc_commit(bar(C::B_DO_EMPTY));
                // phase B of step i done: dP^T(i) read, dS^T(i) in TMEM
                if (!(ok = mbar_wait(bar(C::B_DS_FULL), (uint32_t)(i & 1), abort_flag))) break;
                tc_fence_after();
                if (i + 1 < steps && !(ok = issue_s(i + 1))) break;
                // dK += dS^T Q(i)
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; kk++)
                    mma_ts(tmem + C::COL_DK, tmem + C::COL_PD + 8 * kk, sdesc_sw128(sQ + kk * 2048, C::CB, 1024),
                           ID_DK, (i > 0 || kk > 0) ? 1u : 0u);
                tc_commit(bar(C::B_Q_EMPTY + st));
                tc_commit(bar(C::B_DK_DONE));
            }
            tc_commit(bar(C::B_KDONE));
            if (!ok) mbar_wait_drain(bar(C::B_KDONE), 0, 200000000ull);
        }
    } else if (warp < 8) {
        // ------------------------------- compute (key rows = TMEM lanes, row halves)
        const int hc = warp / 4;
        const int kr = (warp % 4) * 32 + lane;
        const int kj = k0 + kr;
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const bool cap = p.softcap > 0.0f;
        bool ok = true;
        for (int i = 0; i < steps; i++) {
            const int st = i % C::QST;
            const int qb = (m_lo + i % nm) * C::BM;
            if (!(ok = mbar_wait_warp(bar(C::B_Q_FULL + st), (uint32_t)((i / C::QST) & 1), abort_flag))) break;
            if (!(ok = mbar_wait_warp(bar(C::B_S_FULL), (uint32_t)(i & 1), abort_flag))) break;
            tc_fence_after();
            const float *nls = sLSE + st * C::BM;
            const float *nds = sDLT + st * C::BM;
            const bool mask = (k0 + C::BN - 1 > qb) || (W > 0 && k0 <= qb + C::BM - 1 - W);
            // phase A: S^T -> P^T (bf16 pairs) and the dS factors g
            float g[C::HALF / 32][32];
            uint32_t pk[C::HALF / 32][16];
#pragma unroll
            for (int c = 0; c < C::HALF / 32; c++) {
                const int c0 = hc * C::HALF + 32 * c;
                uint32_t sc[32];
                tmem_ld32(tmem + lane_base + C::COL_S + c0, sc);
                tmem_ld_wait(sc);
                if (cap) {
                    if (mask) bwd_p32<true, true>(sc, nls + c0, p, kj, qb + c0, W, pk[c], g[c]);
                    else bwd_p32<true, false>(sc, nls + c0, p, kj, qb + c0, W, pk[c], g[c]);
                } else {
                    if (mask) bwd_p32<false, true>(sc, nls + c0, p, kj, qb + c0, W, pk[c], g[c]);
                    else bwd_p32<false, false>(sc, nls + c0, p, kj, qb + c0, W, pk[c], g[c]);
                }
            }
            // P^T(i) goes over dS^T(i - 1): dK(i - 1) must have read it
            if (i > 0 && !(ok = mbar_wait_warp(bar(C::B_DK_DONE), (uint32_t)((i - 1) & 1), abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < C::HALF / 32; c++)
                tmem_st16(tmem + lane_base + C::COL_PD + hc * (C::HALF / 2) + 16 * c, pk[c]);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_P_FULL));
            // phase B: dP^T -> dS^T (bf16 pairs)
            if (!(ok = mbar_wait_warp(bar(C::B_DP_FULL), (uint32_t)(i & 1), abort_flag))) break;
            tc_fence_after();
            uint32_t dsk[C::HALF / 32][16];
#pragma unroll
            for (int c = 0; c < C::HALF / 32; c++) {
                const int c0 = hc * C::HALF + 32 * c;
                uint32_t dc[32];
                tmem_ld32(tmem + lane_base + C::COL_S + c0, dc);
                tmem_ld_wait(dc);
                bwd_ds32(dc, g[c], nds + c0, p, dsk[c]);
            }
            // dS^T(i) goes over P^T(i): dV(i) must have read it
            if (!(ok = mbar_wait_warp(bar(C::B_DV_DONE), (uint32_t)(i & 1), abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < C::HALF / 32; c++)
                tmem_st16(tmem + lane_base + C::COL_PD + hc * (C::HALF / 2) + 16 * c, dsk[c]);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_DS_FULL));
        }
        // epilogue: this warp's key rows, its half of the dV and of the dK columns
        if (ok) ok = mbar_wait_warp(bar(C::B_KDONE), 0, abort_flag);
        if (ok) {
            tc_fence_after();
            const size_t krow = (size_t)bkv * p.T + (size_t)min(kj, p.T - 1);
            auto store = [&](__nv_bfloat16 *dst_row, uint32_t col, int ncols) {
#pragma unroll 1
                for (int c0 = 0; c0 < ncols; c0 += 32) {
                    uint32_t o[32], w[16];
                    tmem_ld32(tmem + lane_base + col + c0, o);
                    tmem_ld_wait(o);
#pragma unroll
                    for (int e = 0; e < 16; e++) w[e] = pack_bf16x2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1]));
                    if (kj < p.T) {
                        uint4 *dst = reinterpret_cast<uint4 *>(dst_row + c0);
#pragma unroll
                        for (int e = 0; e < 4; e++) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                    }
                }
            };
            store(p.dv + krow * DV + hc * (DV / 2), C::COL_DV + hc * (DV / 2), DV / 2);
            store(p.dk + krow * DK + hc * (DK / 2), C::COL_DK + hc * (DK / 2), DK / 2);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ dQ kernel
struct BwdQParams {
    const float *lse;    // [B*Hq*T]
    const float *delta;  // [B*Hq*T]
    __nv_bfloat16 *dq;   // [B*Hq][T][DK]
    int B, Hq, Hkv, T, window, num_qt;
    float scale, scale_log2, softcap, cap_in, cap_out;  // as in BwdParams
};

template <int DK, int DV>
struct BwdQTc {
    // query rows per CTA, keys per tile, keys per softmax warpgroup (half a tile)
    static constexpr int BM = 128, BN = 128, HB = 64;
    static constexpr int NCBK = DK / 64, NCBV = DV / 64;
    static constexpr uint32_t CB = 128 * 128;             // column block (64 dims) of a 128-row tile
    static constexpr uint32_t TQ = NCBK * CB, TDO = NCBV * CB;
    static constexpr uint32_t TKT = NCBK * CB, TVT = NCBV * CB;
    static constexpr int KST = 2, VST = 1;                // ring slots
    static constexpr uint32_t OFF_Q = 0, OFF_DO = TQ, OFF_K = TQ + TDO, OFF_V = OFF_K + KST * TKT;
    static constexpr uint32_t TILES = OFF_V + VST * TVT;
    static constexpr uint32_t OFF_TMEM_SLOT = 240, OFF_ABORT = 244;
    static constexpr uint32_t CTRL = 256;
    static constexpr uint32_t SMEM = 1024 + TILES + CTRL;
    // warps 0-3 softmax of keys 0-63 of every tile, 4-7 of keys 64-127 (one
    // query row a thread), warp 8 loads Q, dO and the K ring, warp 9 issues MMAs
    // and owns TMEM, warp 10 loads the V ring (so that a V load never waits
    // behind a K load held up by a ring slot that a later dQ product frees).
    // TMEM: two 128-column buffers (S of tile u, then dP over it, then each
    // half's dS over its first 32 columns) for tiles u % 2, and dQ.
    static constexpr int THREADS = 384;
    static constexpr int W_LOAD = 8, W_MMA = 9, W_LOAD_V = 10;
    static constexpr uint32_t COL_DQ = 256;
    static constexpr uint32_t col_buf(int x) { return (uint32_t)(x * BN); }
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_DQ + DK <= TMEM_COLS, "tensor memory");
    static_assert(SMEM <= 232448, "shared memory");
    static constexpr int B_QD = 0, B_K_FULL = 1, B_K_EMPTY = 1 + KST, B_V_FULL = 1 + 2 * KST;
    static constexpr int B_V_EMPTY = B_V_FULL + VST, B_S_FULL = B_V_EMPTY + VST, B_PA = B_S_FULL + 2;
    static constexpr int B_DP_FULL = B_PA + 2, B_DS = B_DP_FULL + 2, B_DQ_DONE = B_DS + 2;
    static constexpr int NBAR = B_DQ_DONE + 1;
    static_assert(NBAR * 8 <= (int)OFF_TMEM_SLOT, "control block");
};

template <int DK, int DV>
__global__ void __launch_bounds__(384, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const BwdQParams p) {
    using C = BwdQTc<DK, DV>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const uint32_t tiles = (sbase + 1023u) & ~1023u;
    const uint32_t ctrl = tiles + C::TILES;
    uint8_t *const ctrl_p = smem_raw + (ctrl - sbase);
    const uint32_t sQ = tiles + C::OFF_Q, sdO = tiles + C::OFF_DO, sK0 = tiles + C::OFF_K, sV0 = tiles + C::OFF_V;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl_p + C::OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctrl_p + C::OFF_TMEM_SLOT);
    auto bar = [&](int i) -> uint32_t { return ctrl + 8u * (uint32_t)i; };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    int qt, bh;
    grouped_block((int)blockIdx.x, p.num_qt, p.B * p.Hq, qt, bh);
    qt = p.num_qt - 1 - qt;  // heaviest tiles first
    const int b = bh / p.Hq, hq = bh % p.Hq;
    const int bkv = b * p.Hkv + hq / (p.Hq / p.Hkv);
    const int W = p.window;
    const int q0 = qt * C::BM;
    const int lo = W > 0 ? max(0, q0 - W + 1) / C::BN : 0;
    const int hi = min(p.T - 1, q0 + C::BM - 1) / C::BN;
    const int n = hi - lo + 1;  // key tiles lo..hi, index u = j - lo

    if (threadIdx.x == 0) {
        mbar_init(bar(C::B_QD), 1);
        for (int s = 0; s < C::KST; s++) {
            mbar_init(bar(C::B_K_FULL + s), 1);
            mbar_init(bar(C::B_K_EMPTY + s), 1);
        }
        for (int s = 0; s < C::VST; s++) {
            mbar_init(bar(C::B_V_FULL + s), 1);
            mbar_init(bar(C::B_V_EMPTY + s), 1);
        }
        for (int x = 0; x < 2; x++) {
            mbar_init(bar(C::B_S_FULL + x), 1);
            mbar_init(bar(C::B_PA + x), 8);
            mbar_init(bar(C::B_DP_FULL + x), 1);
            mbar_init(bar(C::B_DS + x), 8);
        }
        mbar_init(bar(C::B_DQ_DONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::W_LOAD && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
    }
    if (warp == C::W_MMA) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::W_LOAD || warp == C::W_LOAD_V) {
        // ------------------------------------------------------------ producers
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();
            const bool kq = warp == C::W_LOAD;  // Q, dO and K; else V
            if (kq) {
                mbar_arrive_expect_tx(bar(C::B_QD), C::TQ + C::TDO);
                for (int c = 0; c < C::NCBK; c++) tma_load_3d(sQ + c * C::CB, &tmQ, bar(C::B_QD), c * 64, q0, bh);
                for (int c = 0; c < C::NCBV; c++) tma_load_3d(sdO + c * C::CB, &tmdO, bar(C::B_QD), c * 64, q0, bh);
            }
            // K(u) (or V(u)) for u = 0 .. n-1, each ring slot reused once the
            // product that last read it has completed
            const int nst = kq ? C::KST : C::VST;
            const int B_FULL = kq ? C::B_K_FULL : C::B_V_FULL, B_EMPTY = kq ? C::B_K_EMPTY : C::B_V_EMPTY;
            const uint32_t base = kq ? sK0 : sV0, tile = kq ? C::TKT : C::TVT;
            const int ncb = kq ? C::NCBK : C::NCBV;
            const CUtensorMap *map = kq ? &tmK : &tmV;
            int issued = 0;
            bool ok = true;
            for (int u = 0; u < n; u++) {
                const int s = u % nst;
                if (!(ok = mbar_wait(bar(B_EMPTY + s), (uint32_t)(((u / nst) & 1) ^ 1), abort_flag))) break;
                mbar_arrive_expect_tx(bar(B_FULL + s), tile);
                for (int c = 0; c < ncb; c++)
                    tma_load_3d_hint(base + s * tile + c * C::CB, map, bar(B_FULL + s), c * 64, (lo + u) * C::BN, bkv,
                                     keep);
                issued++;
            }
            if (!ok) {
                if (kq) mbar_wait_drain(bar(C::B_QD), 0, 200000000ull);
                for (int back = 1; back <= min(issued, nst); back++) {
                    const int L = issued - back;
                    mbar_wait_drain(bar(B_FULL + L % nst), (uint32_t)((L / nst) & 1), 200000000ull);
                }
            }
        }
    } else if (warp == C::W_MMA) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_bf16_f32(128, C::BN, false, false);
            constexpr uint32_t ID_DQ = idesc_bf16_f32(128, DK, false, true);
            auto offk = [](int kk) -> uint32_t { return (uint32_t)((kk >> 2) * C::CB + (kk & 3) * 32); };
            // S(u) = Q K(u)^T into buffer u % 2
            auto issue_s = [&](int u) -> bool {
                const int s = u % C::KST;
                if (!mbar_wait(bar(C::B_K_FULL + s), (uint32_t)((u / C::KST) & 1), abort_flag)) return false;
                tc_fence_after();
                const uint32_t sK = sK0 + s * C::TKT;
#pragma unroll
                for (int kk = 0; kk < DK / 16; kk++)
                    mma_ss(tmem + C::col_buf(u & 1), sdesc_sw128(sQ + offk(kk), 16, 1024),
                           sdesc_sw128(sK + offk(kk), 16, 1024), ID_S, kk > 0);
                tc_commit(bar(C::B_S_FULL + (u & 1)));
                return true;
            };
            // dP(u) = dO V(u)^T into buffer u % 2 (over S(u), which phase A has read)
            auto issue_dp = [&](int u) -> bool {
                const int s = u % C::VST;
                if (!mbar_wait(bar(C::B_V_FULL + s), (uint32_t)((u / C::VST) & 1), abort_flag)) return false;
                tc_fence_after();
                const uint32_t sV = sV0 + s * C::TVT;
#pragma unroll
                for (int kk = 0; kk < DV / 16; kk++)
                    mma_ss(tmem + C::col_buf(u & 1), sdesc_sw128(sdO + offk(kk), 16, 1024),
                           sdesc_sw128(sV + offk(kk), 16, 1024), ID_S, kk > 0);
                tc_commit(bar(C::B_DP_FULL + (u & 1)));
                tc_commit(bar(C::B_V_EMPTY + s));
                return true;
            };
            // dQ += dS(u) K(u), one half of the keys at a time: dS of half h from
            // the first 32 columns of its 64 in buffer u % 2, K rows 64 h .. MN-major
            // (N = the key head dim)
            auto issue_dq = [&](int u) {
                const int s = u % C::KST;
                const uint32_t sK = sK0 + s * C::TKT;
#pragma unroll
                for (int h = 0; h < 2; h++) {
#pragma unroll
                    for (int kk = 0; kk < C::HB / 16; kk++)
                        mma_ts(tmem + C::COL_DQ, tmem + C::col_buf(u & 1) + C::HB * h + 8 * kk,
                               sdesc_sw128(sK + (h * (C::HB / 16) + kk) * 2048, C::CB, 1024), ID_DQ,
                               (u > 0 || h > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(bar(C::B_K_EMPTY + s));
            };
            // Issue whichever product is ready, each kind in its own order:
            //   S(ns)  once K(ns) has landed and dQ(ns - 2) (the last reader of
            //          buffer ns % 2) has been issued;
            //   dP(np) once S(np) is issued, phase A of tile np is done and V(np)
            //          has landed;
            //   dQ(nq) once dP(nq) is issued and phase B of tile nq is done.
            // S(ns + 1) runs while the softmax warpgroups work on tile ns.
            bool ok = mbar_wait(bar(C::B_QD), 0, abort_flag);
            int ns = 0, np = 0, nq = 0;
            uint64_t t_last = globaltimer_ns();
            while (ok && nq < n) {
                bool progress = false;
                if (nq < np && mbar_try_wait(bar(C::B_DS + (nq & 1)), (uint32_t)((nq >> 1) & 1))) {
                    tc_fence_after();
                    issue_dq(nq++);
                    progress = true;
                }
                if (np < ns && mbar_try_wait(bar(C::B_PA + (np & 1)), (uint32_t)((np >> 1) & 1)) &&
                    mbar_try_wait(bar(C::B_V_FULL + np % C::VST), (uint32_t)((np / C::VST) & 1))) {
                    tc_fence_after();
                    ok = issue_dp(np++);  // its V wait returns at once
                    progress = true;
                }
                if (ok && ns < n && nq >= ns - 1 &&
                    mbar_try_wait(bar(C::B_K_FULL + ns % C::KST), (uint32_t)((ns / C::KST) & 1))) {
                    ok = issue_s(ns++);   // its K wait returns at once
                    progress = true;
                }
                if (progress) {
                    t_last = globaltimer_ns();
                } else if (*abort_flag) {
                    ok = false;
                } else if (globaltimer_ns() - t_last > kWaitLimitNs) {
                    record_status(kStatusTimeout);
                    *abort_flag = 1;
                    ok = false;
                }
            }
            // DQ_DONE fires once every MMA issued so far has completed
            tc_commit(bar(C::B_DQ_DONE));
            if (!ok) mbar_wait_drain(bar(C::B_DQ_DONE), 0, 200000000ull);
        }
    } else if (warp < 8) {
        // --------------- softmax (one query row a thread), keys 64 x .. 64 x + 63 of every tile
        const int x = warp / 4;
        const int row = threadIdx.x % 128;
        const int qi = q0 + row;
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const bool cap = p.softcap > 0.0f;
        const size_t ridx = (size_t)bh * p.T + (size_t)min(qi, p.T - 1);
        // rows past T: P = 0 (and dS = 0) through nl = -inf
        const float nl = qi < p.T ? -p.lse[ridx] * kLog2e : -INFINITY;
        const float nd = qi < p.T ? -p.delta[ridx] * p.scale : 0.0f;
        bool ok = true;
        for (int u = 0; u < n; u++) {
            const int k0 = (lo + u) * C::BN + C::HB * x;
            const uint32_t tB = tmem + lane_base + C::col_buf(u & 1) + C::HB * x;
            const uint32_t ph = (uint32_t)((u >> 1) & 1);  // phase of buffer u % 2's barriers
            if (!(ok = mbar_wait_warp(bar(C::B_S_FULL + (u & 1)), ph, abort_flag))) break;
            tc_fence_after();
            uint32_t s[2][32];
            tmem_ld32(tB, s[0]);
            tmem_ld32(tB + 32, s[1]);
            tmem_ld_wait(s[0]);
            tmem_ld_wait(s[1]);
            // warp-uniform: does any key of the tile fall outside some row's range?
            const int r0 = q0 + 32 * (warp % 4);
            const bool mask = (k0 + C::HB - 1 > r0) || (W > 0 && k0 <= r0 + 31 - W);
            float g[2][32];
#pragma unroll
            for (int h = 0; h < 2; h++) {
#pragma unroll
                for (int c = 0; c < 32; c++) {
                    const float v = __uint_as_float(s[h][c]);
                    float pr, gg;
                    if (cap) {
                        const float t = tanh_via_ex2(v * p.cap_in);
                        pr = ex2_approx(fmaf(p.cap_out, t, nl));
                        gg = pr * (1.0f - t * t);
                    } else {
                        pr = ex2_approx(fmaf(v, p.scale_log2, nl));
                        gg = pr;
                    }
                    if (mask) {
                        const int kj = k0 + 32 * h + c;
                        const bool vis = kj <= qi && (W == 0 || kj > qi - W);
                        gg = vis ? gg : 0.0f;
                    }
                    g[h][c] = gg;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_PA + (u & 1)));
            // phase B: dP -> dS (bf16) into the buffer's first 32 columns
            if (!(ok = mbar_wait_warp(bar(C::B_DP_FULL + (u & 1)), ph, abort_flag))) break;
            tc_fence_after();
            uint32_t d[2][32];
            tmem_ld32(tB, d[0]);
            tmem_ld32(tB + 32, d[1]);
            tmem_ld_wait(d[0]);
            tmem_ld_wait(d[1]);
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; c++) {
                const int a = 2 * c;
                const float d0 = g[a >> 5][a & 31] * fmaf(__uint_as_float(d[a >> 5][a & 31]), p.scale, nd);
                const float d1 = g[(a + 1) >> 5][(a + 1) & 31] * fmaf(__uint_as_float(d[(a + 1) >> 5][(a + 1) & 31]), p.scale, nd);
                pk[c] = pack_bf16x2(d0, d1);
            }
            tmem_st32(tB, pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_DS + (u & 1)));
        }
        // epilogue: warpgroup x writes its half of the dQ columns of its rows
        if (ok) ok = mbar_wait_warp(bar(C::B_DQ_DONE), 0, abort_flag);
        if (ok) {
            tc_fence_after();
            __nv_bfloat16 *drow = p.dq + ((size_t)bh * p.T + (size_t)min(qi, p.T - 1)) * DK + x * (DK / 2);
#pragma unroll 1
            for (int c0 = 0; c0 < DK / 2; c0 += 32) {
                uint32_t o[32], w[16];
                tmem_ld32(tmem + lane_base + C::COL_DQ + x * (DK / 2) + c0, o);
                tmem_ld_wait(o);
#pragma unroll
                for (int e = 0; e < 16; e++) w[e] = pack_bf16x2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1]));
                if (qi < p.T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(drow + c0);
#pragma unroll
                    for (int e = 0; e < 4; e++) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace forge
