// bwd_tc.cuh -- tensor-core backward main kernel (bf16 in, f32 accumulate).
//
// One CTA per (KV tile of 128 keys, batch, KV head, head-dim half). The CTA keeps
// its K and V tiles in shared memory and dK, dV accumulators in tensor memory for
// the whole run, and walks every (query head of the group, query tile) pair that
// can see its keys: query tiles from the key tile's diagonal up to the window's
// reach (or T - 1), so the cost scales with the window. Per step i:
//   S^T  = K Q^T            (tcgen05, 128 x BM, f32 in TMEM)
//   dP^T = V dO^T           (tcgen05)
//   P^T  = exp2(s*log2e - LSE*log2e), masked to 0   -> bf16 into TMEM (over S^T)
//   dS^T = scale * P^T (dP^T - Delta) [* (1 - tanh^2)] -> bf16 into shared memory
//          (the cap factor is the "exact tanh' chain": src/nn/attention.h
//           commit log, Wave 2)
//   dV  += P^T dO           (A from TMEM)
//   dK  += dS^T Q
//   dQ   = dS K  (or its transpose K^T dS^T), drained from TMEM by four warps
//          into a swizzled f32 staging tile in shared memory and added into a
//          padded [B*Hq][Tpad][D] f32 workspace with TMA bulk reduce-add (head
//          dim 256, which has no shared memory left for staging, adds with
//          per-element f32 reductions instead).
// dK and dV sum over the group's query heads inside the CTA, so they need no
// atomics; dQ rows are shared between key tiles and are reduced in L2.
//
// Overlap (head dim 128): S^T and dS^T are double-buffered and the compute warps
// copy dP^T into registers as soon as it lands, so the MMA warp issues
// S^T(i+1) and dP^T(i+1) while step i's P and dS are being formed, and step
// i+1's P/dS math runs while dV, dK, dQ of step i are on the tensor cores.
//
// Shapes per head dim (TMEM columns: NSB x S^T + dP^T + dV + dK + dQ <= 512):
//   D = 64 : BM = 128 query rows, one S buffer, dQ = dS K (M = 128 rows, N = 64)
//   D = 128: BM = 64, two S buffers, dQ^T = K^T dS^T (M = 128 = D, N = 64 rows)
//   D = 256: BM = 64, one S buffer, two CTAs per key tile, each owning half of
//            the head dim (DH = 128) for dK, dV and dQ; S^T and dP^T use the
//            full head dim.
//
// Roles (320 threads): warps 0-3 compute (one thread per key row, TMEM lane),
// warps 4-7 dQ drain + dK epilogue, warp 8 loads (TMA for tiles, plain loads
// for LSE and Delta), warp 9 issues MMAs and owns TMEM.
#pragma once

#include "sm100.cuh"

namespace forge {

template <int D_>
struct BwdTc {
    static constexpr int D = D_;
    static constexpr int BN = 128;                       // keys per CTA
    static constexpr int BM = D == 64 ? 128 : 64;        // query rows per step
    static constexpr bool DQT = D != 64;                 // transposed dQ product
    static constexpr int NSPLIT = D == 256 ? 2 : 1;      // head-dim halves
    static constexpr int DH = D / NSPLIT;                // output columns per CTA
    static constexpr int QST = D == 256 ? 1 : (D == 128 ? 3 : 2);  // Q/dO stages
    static constexpr int NSB = D == 128 ? 2 : 1;         // S^T / dS^T buffers
    static constexpr bool PRELOAD = (BM == 64);          // whole S^T/dP^T rows in registers
    static constexpr int NCB = D / 64;
    static constexpr uint32_t CBK = 128 * 128;           // column block of a 128-row tile
    static constexpr uint32_t CBQ = BM * 128;            // column block of a BM-row tile
    static constexpr uint32_t TK = NCB * CBK;            // K (or V) tile bytes
    static constexpr uint32_t TQ = NCB * CBQ;            // Q (or dO) tile bytes
    static constexpr uint32_t TS = (BM / 64) * CBK;      // dS^T tile bytes
    static constexpr uint32_t OFF_K = 0, OFF_V = TK, OFF_Q = 2 * TK;
    static constexpr uint32_t OFF_DO = OFF_Q + QST * TQ;
    static constexpr uint32_t OFF_DS = OFF_DO + QST * TQ;
    static constexpr bool BULK_DQ = D != 256;            // staged TMA reduce-add of dQ
    static constexpr int NSTG = D == 64 ? 2 : 1;         // dQ staging tiles
    static constexpr uint32_t STG = BM * DH * 4;         // one f32 dQ staging tile
    static constexpr uint32_t OFF_STG = OFF_DS + NSB * TS;
    static constexpr uint32_t TILES = OFF_STG + (BULK_DQ ? NSTG * STG : 0);
    // control block: barriers, TMEM slot, abort flag, per-stage LSE/Delta rows
    static constexpr uint32_t OFF_TMEM_SLOT = 240, OFF_ABORT = 244;
    static constexpr uint32_t OFF_LSE = 256;                        // [QST][BM] f32, LSE * log2(e)
    static constexpr uint32_t OFF_DLT = OFF_LSE + QST * BM * 4;     // [QST][BM] f32, scale * Delta
    static constexpr uint32_t CTRL = (OFF_DLT + QST * BM * 4 + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM = CTRL + TILES + 1024;
    static constexpr int THREADS = 320;
    static constexpr uint32_t COL_DP = NSB * BM, COL_DV = COL_DP + BM, COL_DK = COL_DV + DH;
    static constexpr uint32_t COL_DQ = COL_DK + DH;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t col_s(int b) { return (uint32_t)(b * BM); }
    static_assert(COL_DQ + (DQT ? BM : DH) <= 512, "tensor memory");
    static_assert(!DQT || DH == 128, "transposed dQ needs M = 128");
    static_assert(SMEM <= 232448, "shared memory");
    // barriers
    static constexpr int B_KV = 0;
    static constexpr int B_Q_FULL = 1;                   // [QST]
    static constexpr int B_Q_EMPTY = B_Q_FULL + QST;     // [QST]
    static constexpr int B_S_FULL = B_Q_EMPTY + QST;     // [NSB]
    static constexpr int B_DS_EMPTY = B_S_FULL + NSB;    // [NSB]
    static constexpr int B_PDS_FULL = B_DS_EMPTY + NSB;  // [NSB] P^T and dS^T of a buffer ready
    static constexpr int B_DP_FULL = B_PDS_FULL + NSB;
    static constexpr int B_DP_FREE = B_DP_FULL + 1;
    static constexpr int B_DQ_FULL = B_DP_FREE + 1;
    static constexpr int B_DQ_FREE = B_DQ_FULL + 1;
    static constexpr int B_KDONE = B_DQ_FREE + 1;
    static constexpr int NBAR = B_KDONE + 1;
    static_assert(NBAR * 8 <= (int)OFF_TMEM_SLOT, "control block");
};

struct BwdParams {
    const float *lse;      // [B*Hq*T]
    const float *delta;    // [B*Hq*T]
    float *dq_acc;         // [B*Hq][Tpad][D]
    __nv_bfloat16 *dk, *dv;
    int B, Hq, Hkv, T, Tpad, window, num_kt;
    float scale;           // softmax scale (folded into dS)
    float scale_log2;      // scale * log2(e)
    float softcap;         // 0 = off
    float cap_in;          // scale / softcap
    float cap_out;         // softcap * log2(e)
};

// P and dS for 32 query columns of one key row (this thread's TMEM lane).
//   s, dp : raw S^T and dP^T accumulators of the 32 columns
//   l2, dl: LSE*log2(e) and scale*Delta of the 32 columns
//   pk, dk: bf16x2-packed P^T and dS^T (column pairs, low half = even column)
// CAP and MASK are compile-time so the unrolled loop is one basic block.
template <bool CAP, bool MASK>
__device__ __forceinline__ void bwd_math32(const uint32_t (&s)[32], const uint32_t (&dp)[32], const float *l2s,
                                           const float *dls, const BwdParams &p, int kj, int q0, int W,
                                           uint32_t (&pk)[16], uint32_t (&dk)[16]) {
    float l2[4], dl[4];
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
        if ((c & 3) == 0) {
            const float4 a = *reinterpret_cast<const float4 *>(l2s + c);
            const float4 d4 = *reinterpret_cast<const float4 *>(dls + c);
            l2[0] = a.x; l2[1] = a.y; l2[2] = a.z; l2[3] = a.w;
            dl[0] = d4.x; dl[1] = d4.y; dl[2] = d4.z; dl[3] = d4.w;
        }
        float pp[2], dd[2];
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const float x = __uint_as_float(s[c + e]);
            float pr, g;
            // a quarter of the exponentials on the FMA pipe when nothing is masked
            const bool emu = !MASK && (c & 6) == 6;
            if constexpr (CAP) {
                const float t = tanh_via_ex2(x * p.cap_in);
                const float y = fmaf(p.cap_out, t, -l2[(c & 3) + e]);
                pr = emu ? exp2_poly(y) : ex2_approx(y);
                g = pr * (1.0f - t * t);
            } else {
                const float y = fmaf(x, p.scale_log2, -l2[(c & 3) + e]);
                pr = emu ? exp2_poly(y) : ex2_approx(y);
                g = pr;
            }
            if constexpr (MASK) {
                const int qi = q0 + c + e;
                const bool vis = kj <= qi && (W == 0 || kj > qi - W);
                pr = vis ? pr : 0.0f;
                g = vis ? g : 0.0f;
            }
            pp[e] = pr;
            dd[e] = g * fmaf(__uint_as_float(dp[c + e]), p.scale, -dl[(c & 3) + e]);
        }
        pk[c >> 1] = pack_bf16x2(pp[0], pp[1]);
        dk[c >> 1] = pack_bf16x2(dd[0], dd[1]);
    }
}

// One 32-column chunk: LSE/Delta terms from shared memory, P/dS math, P^T into
// TMEM (columns [c0/2, c0/2 + 16) of the S buffer, already read), dS^T into the
// swizzled shared-memory tile (row kr, 16-byte chunk index XOR row % 8).
template <int D>
__device__ __forceinline__ void bwd_chunk(const uint32_t (&s)[32], const uint32_t (&dp)[32], const float *l2s,
                                          const float *dls, const BwdParams &p, bool cap, bool mask, int kj, int q0,
                                          int W, int c0, int kr, uint32_t tS, uint32_t sdS) {
    using C = BwdTc<D>;
    const float *l2 = l2s + c0, *dl = dls + c0;
    uint32_t pk[16], dk[16];
    if (cap) {
        if (mask) bwd_math32<true, true>(s, dp, l2, dl, p, kj, q0, W, pk, dk);
        else bwd_math32<true, false>(s, dp, l2, dl, p, kj, q0, W, pk, dk);
    } else {
        if (mask) bwd_math32<false, true>(s, dp, l2, dl, p, kj, q0, W, pk, dk);
        else bwd_math32<false, false>(s, dp, l2, dl, p, kj, q0, W, pk, dk);
    }
    tmem_st16(tS + (uint32_t)(c0 >> 1), pk);
    const uint32_t blk = sdS + (uint32_t)(c0 >> 6) * C::CBK + (uint32_t)kr * 128u;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const uint32_t chunk = (uint32_t)(((c0 & 63) >> 3) + e);
        const uint32_t addr = blk + ((chunk ^ (uint32_t)(kr & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dk[4 * e]), "r"(dk[4 * e + 1]),
                     "r"(dk[4 * e + 2]), "r"(dk[4 * e + 3])
                     : "memory");
    }
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmAcc, const BwdParams p) {
    using C = BwdTc<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const uint32_t tiles = (sbase + C::CTRL + 1023u) & ~1023u;
    const uint32_t sK = tiles + C::OFF_K, sV = tiles + C::OFF_V, sQ0 = tiles + C::OFF_Q;
    const uint32_t sdO0 = tiles + C::OFF_DO, sdS0 = tiles + C::OFF_DS, sStg = tiles + C::OFF_STG;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem_raw + C::OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + C::OFF_TMEM_SLOT);
    float *sLSE = reinterpret_cast<float *>(smem_raw + C::OFF_LSE);
    float *sDLT = reinterpret_cast<float *>(smem_raw + C::OFF_DLT);
    auto bar = [&](int i) -> uint32_t { return sbase + 8u * (uint32_t)i; };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // work item: key tile n (heaviest = smallest n first), batch b, KV head, half h
    const int per_n = p.B * p.Hkv * C::NSPLIT;
    const int n = blockIdx.x / per_n;
    int rest = blockIdx.x % per_n;
    const int h = rest % C::NSPLIT;
    rest /= C::NSPLIT;
    const int bkv = rest;  // b * Hkv + hkv
    const int b = bkv / p.Hkv, hkv = bkv % p.Hkv;
    const int G = p.Hq / p.Hkv;
    const int k0 = n * C::BN;
    const int W = p.window;
    const int m_lo = k0 / C::BM;
    const int q_last = W > 0 ? min(p.T - 1, k0 + C::BN - 1 + W - 1) : p.T - 1;
    const int m_hi = q_last / C::BM;
    const int nm = m_hi - m_lo + 1;
    const int steps = G * nm;

    if (threadIdx.x == 0) {
        mbar_init(bar(C::B_KV), 1);
        for (int s = 0; s < C::QST; s++) {
            mbar_init(bar(C::B_Q_FULL + s), 33);
            mbar_init(bar(C::B_Q_EMPTY + s), 1);
        }
        for (int s = 0; s < C::NSB; s++) {
            mbar_init(bar(C::B_S_FULL + s), 1);
            mbar_init(bar(C::B_DS_EMPTY + s), 1);
            mbar_init(bar(C::B_PDS_FULL + s), 4);
        }
        mbar_init(bar(C::B_DP_FULL), 1);
        mbar_init(bar(C::B_DP_FREE), 4);
        mbar_init(bar(C::B_DQ_FULL), 1);
        mbar_init(bar(C::B_DQ_FREE), 4);
        mbar_init(bar(C::B_KDONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmAcc);
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ producer
        int issued = 0;
        bool ok = true;
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::TK);
            for (int c = 0; c < C::NCB; c++) {
                tma_load_3d(sK + c * C::CBK, &tmK, bar(C::B_KV), c * 64, k0, bkv);
                tma_load_3d(sV + c * C::CBK, &tmV, bar(C::B_KV), c * 64, k0, bkv);
            }
        }
        for (int i = 0; i < steps; i++) {
            const int st = i % C::QST;
            const uint32_t ph = (uint32_t)((i / C::QST) & 1);
            const int g = i / nm, m = m_lo + i % nm;
            const int bhq = b * p.Hq + hkv * G + g;
            // this step's LSE and Delta into registers first: their global-load
            // latency overlaps the wait for a free stage
            float lv[C::BM / 32], dv[C::BM / 32];
#pragma unroll
            for (int r = 0; r < C::BM / 32; r++) {
                const int q = m * C::BM + lane + 32 * r;
                const size_t idx = (size_t)bhq * p.T + (size_t)min(q, p.T - 1);
                lv[r] = q < p.T ? p.lse[idx] * kLog2e : INFINITY;
                dv[r] = q < p.T ? p.delta[idx] * p.scale : 0.0f;
            }
            if (!mbar_wait_warp(bar(C::B_Q_EMPTY + st), ph ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(C::B_Q_FULL + st), 2 * C::TQ);
                for (int c = 0; c < C::NCB; c++) {
                    tma_load_3d(sQ0 + st * C::TQ + c * C::CBQ, &tmQ, bar(C::B_Q_FULL + st), c * 64, m * C::BM, bhq);
                    tma_load_3d(sdO0 + st * C::TQ + c * C::CBQ, &tmdO, bar(C::B_Q_FULL + st), c * 64, m * C::BM,
                                bhq);
                }
            }
            issued++;
#pragma unroll
            for (int r = 0; r < C::BM / 32; r++) {
                sLSE[st * C::BM + lane + 32 * r] = lv[r];
                sDLT[st * C::BM + lane + 32 * r] = dv[r];
            }
            mbar_arrive(bar(C::B_Q_FULL + st));
        }
        if (!ok && lane == 0) {
            mbar_wait_drain(bar(C::B_KV), 0, 200000000ull);
            for (int back = 1; back <= min(issued, C::QST); back++) {
                const int L = issued - back;
                mbar_wait_drain(bar(C::B_Q_FULL + L % C::QST), (uint32_t)((L / C::QST) & 1), 200000000ull);
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_bf16_f32(128, C::BM, false, false);
            constexpr uint32_t ID_ACC = idesc_bf16_f32(128, C::DH, false, true);
            constexpr uint32_t ID_DQ =
                C::DQT ? idesc_bf16_f32(128, C::BM, true, true) : idesc_bf16_f32(128, C::D, true, true);
            const uint32_t h_q = (uint32_t)h * (C::DH / 64) * C::CBQ;  // column-block offset of half h
            const uint32_t h_k = (uint32_t)h * (C::DH / 64) * C::CBK;
            // S^T(j) = K Q(j)^T into S buffer j % NSB, over the full head dim
            auto issue_s = [&](int j) -> bool {
                const int st = j % C::QST;
                if (!mbar_wait(bar(C::B_Q_FULL + st), (uint32_t)((j / C::QST) & 1), abort_flag)) return false;
                tc_fence_after();
                const uint32_t sQ = sQ0 + st * C::TQ;
                const uint32_t dS = tmem + C::col_s(j % C::NSB);
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++) {
                    const uint32_t ok_ = (kk >> 2) * C::CBK + (kk & 3) * 32;
                    const uint32_t oq = (kk >> 2) * C::CBQ + (kk & 3) * 32;
                    mma_ss(dS, sdesc_sw128(sK + ok_, 16, 1024), sdesc_sw128(sQ + oq, 16, 1024), ID_S, kk > 0);
                }
                tc_commit(bar(C::B_S_FULL + j % C::NSB));
                return true;
            };
            // dP^T(j) = V dO(j)^T (the stage of j is already known to be full)
            auto issue_dp = [&](int j) {
                const uint32_t sdO = sdO0 + (j % C::QST) * C::TQ;
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++) {
                    const uint32_t ok_ = (kk >> 2) * C::CBK + (kk & 3) * 32;
                    const uint32_t oq = (kk >> 2) * C::CBQ + (kk & 3) * 32;
                    mma_ss(tmem + C::COL_DP, sdesc_sw128(sV + ok_, 16, 1024), sdesc_sw128(sdO + oq, 16, 1024), ID_S,
                           kk > 0);
                }
                tc_commit(bar(C::B_DP_FULL));
            };
            bool ok = mbar_wait(bar(C::B_KV), 0, abort_flag);
            if (ok && (ok = issue_s(0))) issue_dp(0);
            for (int i = 0; ok && i < steps; i++) {
                const int st = i % C::QST, sb = i % C::NSB;
                const uint32_t sQ = sQ0 + st * C::TQ, sdO = sdO0 + st * C::TQ, sdS = sdS0 + sb * C::TS;
                const bool more = i + 1 < steps;
                if (C::NSB == 2 && more) {
                    // next step's products while this step's P and dS are formed
                    if (!(ok = issue_s(i + 1))) break;
                    if (!(ok = mbar_wait(bar(C::B_DP_FREE), (uint32_t)(i & 1), abort_flag))) break;
                    issue_dp(i + 1);
                }
                if (!(ok = mbar_wait(bar(C::B_PDS_FULL + sb), (uint32_t)((i / C::NSB) & 1), abort_flag))) break;
                tc_fence_after();
                // dV += P^T dO (P^T from TMEM), dK += dS^T Q
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; kk++)
                    mma_ts(tmem + C::COL_DV, tmem + C::col_s(sb) + kk * 8,
                           sdesc_sw128(sdO + h_q + kk * 2048, C::CBQ, 1024), ID_ACC, (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; kk++) {
                    const uint32_t oa = (kk >> 2) * C::CBK + (kk & 3) * 32;
                    mma_ss(tmem + C::COL_DK, sdesc_sw128(sdS + oa, 16, 1024),
                           sdesc_sw128(sQ + h_q + kk * 2048, C::CBQ, 1024), ID_ACC, (i > 0 || kk > 0) ? 1u : 0u);
                }
                // dQ (the drain warps must have emptied the previous one)
                if (i > 0) {
                    if (!(ok = mbar_wait(bar(C::B_DQ_FREE), (uint32_t)((i - 1) & 1), abort_flag))) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; kk++) {
                    if constexpr (C::DQT) {
                        mma_ss(tmem + C::COL_DQ, sdesc_sw128(sK + h_k + kk * 2048, C::CBK, 1024),
                               sdesc_sw128(sdS + kk * 2048, C::CBK, 1024), ID_DQ, kk > 0);
                    } else {
                        mma_ss(tmem + C::COL_DQ, sdesc_sw128(sdS + kk * 2048, C::CBK, 1024),
                               sdesc_sw128(sK + kk * 2048, C::CBK, 1024), ID_DQ, kk > 0);
                    }
                }
                tc_commit(bar(C::B_DQ_FULL));
                tc_commit(bar(C::B_Q_EMPTY + st));
                tc_commit(bar(C::B_DS_EMPTY + sb));
                if (C::NSB == 1 && more) {
                    if (!(ok = issue_s(i + 1))) break;
                    issue_dp(i + 1);
                }
            }
            tc_commit(bar(C::B_KDONE));
            if (!ok) mbar_wait_drain(bar(C::B_KDONE), 0, 200000000ull);
        }
    } else if (warp < 4) {
        // ------------------------------------------- compute (key rows, TMEM lanes)
        const int kr = threadIdx.x;  // key row within the tile
        const int kj = k0 + kr;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const bool cap = p.softcap > 0.0f;
        bool ok = true;
        for (int i = 0; i < steps; i++) {
            const int st = i % C::QST, sb = i % C::NSB;
            const int m = m_lo + i % nm;
            const int qb = m * C::BM;
            if (!(ok = mbar_wait_warp(bar(C::B_Q_FULL + st), (uint32_t)((i / C::QST) & 1), abort_flag))) break;
            if (!(ok = mbar_wait_warp(bar(C::B_S_FULL + sb), (uint32_t)((i / C::NSB) & 1), abort_flag))) break;
            if (!(ok = mbar_wait_warp(bar(C::B_DP_FULL), (uint32_t)(i & 1), abort_flag))) break;
            tc_fence_after();
            const uint32_t tS = tmem + lane_base + C::col_s(sb);
            const uint32_t tP = tmem + lane_base + C::COL_DP;
            const float *l2s = sLSE + st * C::BM;
            const float *dls = sDLT + st * C::BM;
            const uint32_t sdS = sdS0 + sb * C::TS;
            const bool mask = (k0 + C::BN - 1 > qb) || (W > 0 && k0 <= qb + C::BM - 1 - W);
            if constexpr (C::PRELOAD) {
                // the whole dP^T row (64 columns) into registers: dP^T is then free
                // for the next step's product; S^T is read chunk by chunk
                uint32_t d0[32], d1[32];
                tmem_ld32(tP, d0);
                tmem_ld32(tP + 32, d1);
                tmem_ld_wait(d0);
                tmem_ld_wait(d1);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_DP_FREE));
                // dS^T buffer sb was last read by the dK/dQ products of step i - NSB
                if (i >= C::NSB &&
                    !(ok = mbar_wait_warp(bar(C::B_DS_EMPTY + sb), (uint32_t)(((i / C::NSB) - 1) & 1), abort_flag)))
                    break;
                {
                    uint32_t sc[32];
                    tmem_ld32(tS, sc);
                    tmem_ld_wait(sc);
                    bwd_chunk<D>(sc, d0, l2s, dls, p, cap, mask, kj, qb, W, 0, kr, tS, sdS);
                }
                {
                    uint32_t sc[32];
                    tmem_ld32(tS + 32, sc);
                    tmem_ld_wait(sc);
                    bwd_chunk<D>(sc, d1, l2s, dls, p, cap, mask, kj, qb + 32, W, 32, kr, tS, sdS);
                }
            } else {
                if (i >= C::NSB &&
                    !(ok = mbar_wait_warp(bar(C::B_DS_EMPTY + sb), (uint32_t)(((i / C::NSB) - 1) & 1), abort_flag)))
                    break;
#pragma unroll 1
                for (int c0 = 0; c0 < C::BM; c0 += 32) {
                    uint32_t sc[32], dc[32];
                    tmem_ld32(tS + c0, sc);
                    tmem_ld32(tP + c0, dc);
                    tmem_ld_wait(sc);
                    tmem_ld_wait(dc);
                    bwd_chunk<D>(sc, dc, l2s, dls, p, cap, mask, kj, qb + c0, W, c0, kr, tS, sdS);
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (!C::PRELOAD) mbar_arrive(bar(C::B_DP_FREE));
                mbar_arrive(bar(C::B_PDS_FULL + sb));
            }
        }
        // epilogue: dV rows
        if (ok) ok = mbar_wait_warp(bar(C::B_KDONE), 0, abort_flag);
        if (ok) {
            tc_fence_after();
            __nv_bfloat16 *row = p.dv + ((size_t)bkv * p.T + (size_t)min(kj, p.T - 1)) * D + h * C::DH;
#pragma unroll 1
            for (int c0 = 0; c0 < C::DH; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + C::COL_DV + c0, o);
                tmem_ld_wait(o);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; i++) w[i] = pack_bf16x2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1]));
                if (kj < p.T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(row + c0);
#pragma unroll
                    for (int i = 0; i < 4; i++) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
        }
    } else {
        // ------------------------------------ dQ drain (warps 4..7), dK epilogue
        const int t = threadIdx.x - 128;  // TMEM lane of this thread
        const uint32_t lane_base = (uint32_t)((warp - 4) * 32) << 16;
        bool ok = true;
        for (int i = 0; i < steps; i++) {
            const int g = i / nm, m = m_lo + i % nm;
            const int bhq = b * p.Hq + hkv * G + g;
            if (!(ok = mbar_wait_warp(bar(C::B_DQ_FULL), (uint32_t)(i & 1), abort_flag))) break;
            tc_fence_after();
            // two 32-column TMEM loads: this thread's 64 dQ values
            uint32_t v0[32], v1[32];
            tmem_ld32(tmem + lane_base + C::COL_DQ, v0);
            tmem_ld32(tmem + lane_base + C::COL_DQ + 32, v1);
            tmem_ld_wait(v0);
            tmem_ld_wait(v1);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_DQ_FREE));
            if constexpr (C::BULK_DQ) {
                // Staging tile [BM rows][DH cols] f32, stored as DH/32 column blocks of
                // [BM][32] with the 128-byte swizzle (16-byte chunk ^ row % 8), the
                // layout of a TMA box {32, BM, 1}. The tile is reused once the reduce
                // that last read it (NSTG steps ago) has read its source.
                const uint32_t stg = sStg + (uint32_t)(i % C::NSTG) * C::STG;
                if (t == 0) bulk_wait_read<C::NSTG - 1>();
                named_barrier_sync(1, 128);
                if constexpr (C::DQT) {
                    // thread t = head-dim column t of this half; v = 64 query rows
                    const uint32_t cb = (uint32_t)t >> 5, ch = ((uint32_t)t & 31u) >> 2, w4 = ((uint32_t)t & 3u) << 2;
                    const uint32_t base = stg + cb * (uint32_t)(C::BM * 128) + w4;
#pragma unroll
                    for (int c = 0; c < 32; c++) {
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(base + (uint32_t)c * 128u + ((ch ^ ((uint32_t)c & 7u)) << 4)),
                                     "r"(v0[c]) : "memory");
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(base + (uint32_t)(c + 32) * 128u +
                                                                     ((ch ^ ((uint32_t)(c + 32) & 7u)) << 4)),
                                     "r"(v1[c]) : "memory");
                    }
                } else {
                    // thread t = query row t; v = the 64 head-dim values of that row
                    const uint32_t row = stg + (uint32_t)t * 128u;
#pragma unroll
                    for (int c4 = 0; c4 < 8; c4++) {
                        const uint32_t sw = (((uint32_t)c4 ^ ((uint32_t)t & 7u)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + sw), "r"(v0[4 * c4]),
                                     "r"(v0[4 * c4 + 1]), "r"(v0[4 * c4 + 2]), "r"(v0[4 * c4 + 3]) : "memory");
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + (uint32_t)(C::BM * 128) + sw),
                                     "r"(v1[4 * c4]), "r"(v1[4 * c4 + 1]), "r"(v1[4 * c4 + 2]), "r"(v1[4 * c4 + 3])
                                     : "memory");
                    }
                }
                fence_proxy_async_smem();
                named_barrier_sync(1, 128);
                if (t == 0) {
#pragma unroll
                    for (int cb = 0; cb < C::DH / 32; cb++)
                        tma_reduce_add_3d(&tmAcc, stg + (uint32_t)cb * (uint32_t)(C::BM * 128), h * C::DH + 32 * cb,
                                          m * C::BM, bhq);
                    bulk_commit();
                }
            } else {
                // head dim 256: lane = head-dim column h*DH + t, 64 query rows
                float *base = p.dq_acc + ((size_t)bhq * p.Tpad + (size_t)m * C::BM) * D + h * C::DH + t;
#pragma unroll
                for (int c = 0; c < 32; c++) {
                    atomicAdd(base + (size_t)c * D, __uint_as_float(v0[c]));
                    atomicAdd(base + (size_t)(c + 32) * D, __uint_as_float(v1[c]));
                }
            }
        }
        if constexpr (C::BULK_DQ) {
            if (t == 0) bulk_wait<0>();  // reductions complete before the CTA retires
        }
        if (ok) ok = mbar_wait_warp(bar(C::B_KDONE), 0, abort_flag);
        if (ok) {
            tc_fence_after();
            const int kj = k0 + t;
            __nv_bfloat16 *row = p.dk + ((size_t)bkv * p.T + (size_t)min(kj, p.T - 1)) * D + h * C::DH;
#pragma unroll 1
            for (int c0 = 0; c0 < C::DH; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + C::COL_DK + c0, o);
                tmem_ld_wait(o);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; i++) w[i] = pack_bf16x2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1]));
                if (kj < p.T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(row + c0);
#pragma unroll
                    for (int i = 0; i < 4; i++) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace forge
