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
//          (the cap's derivative taken exactly, as every backward on the pages
//           does: src/nn/attention.h commit log, Wave 2)
//   dV  += P^T dO           (A from TMEM)
//   dK  += dS^T Q
//   dQ   = dS K  (or its transpose K^T dS^T), drained from TMEM by four warps
//          and added into a padded [B*Hq][Tpad][D] f32 workspace: head dim 64
//          through a swizzled f32 staging tile in shared memory and TMA bulk
//          reduce-add; head dims 128 and 256, which have no shared memory left
//          for staging, with warp-coalesced f32 reductions from registers.
// dK and dV sum over the group's query heads inside the CTA, so they need no
// atomics; dQ rows are shared between key tiles and are reduced in L2.
//
// Steps of 128 query rows keep every product at N = 128 (or M = N = 128 for
// dQ^T): a tcgen05.mma with both operands in shared memory reads A and B
// (4 KB + N/32 KB per K = 16 slice) at the shared-memory port's rate, so
// narrower products are bound by that port rather than by the tensor cores.
//
// Shapes per head dim (TMEM columns: S^T + dP^T + dV + dK (+ dQ) <= 512):
//   D = 64 : BM = 128 query rows, dQ = dS K (M = 128 rows, N = 64)
//   D = 128: BM = 128, dQ^T = K^T dS^T (M = 128 = D, N = 128 rows) in the
//            columns of dP^T (already copied to registers when dQ^T is issued;
//            dP^T of the next step waits until the drain warps copied dQ^T)
//   D = 256: BM = 64, two CTAs per key tile, each owning half of the head dim
//            (DH = 128) for dK, dV and dQ; S^T and dP^T use the full head dim.
//
// Each step runs in two phases on the compute warps: phase A (needs S^T) forms
// P^T into TMEM and keeps the factors of dS in registers; phase B (needs dP^T)
// forms dS^T into shared memory. The MMA warp issues dV(i) as soon as phase A
// of step i ends and S^T(i + 1) right after it, so S^T(i + 1) and dV(i) run
// during phase B, and dP^T(i + 1) during phase A of step i + 1.
//
// Roles (512 threads): warps 0-7 compute (warp w: key rows = TMEM lanes
// 32 (w % 4).., query-row half w / 4 of the step; they also write each item's
// dV rows, except at head dim 64), warps 8-11 dQ drain + dK epilogue (+ dV at
// head dim 64), warp 12 loads (TMA for tiles, plain loads for LSE and Delta),
// warp 13 issues MMAs and owns TMEM, warps 14-15 idle (see BwdTc for the
// register split).
#pragma once

#include "sm100.cuh"

namespace forge {

template <int D_>
struct BwdTc {
    static constexpr int D = D_;
    static constexpr int BN = 128;                       // keys per CTA
    static constexpr int BM = D == 256 ? 64 : 128;       // query rows per step
    static constexpr bool DQT = D != 64;                 // transposed dQ product
    static constexpr int NSPLIT = D == 256 ? 2 : 1;      // head-dim halves
    static constexpr int DH = D / NSPLIT;                // output columns per CTA
    static constexpr int QST = D == 256 ? 1 : 2;         // Q/dO stages
    // head dim 128: dQ^T takes the TMEM columns of dP^T, which the compute warps
    // have copied out by the time dQ^T is issued (dP^T of the next step then
    // waits for the drain warps to copy dQ^T out)
    static constexpr bool DQ_ALIAS = D == 128;
    static constexpr int NCB = D / 64;
    static constexpr uint32_t CBK = 128 * 128;           // column block of a 128-row tile
    static constexpr uint32_t CBQ = BM * 128;            // column block of a BM-row tile
    static constexpr uint32_t TK = NCB * CBK;            // K (or V) tile bytes
    static constexpr uint32_t TQ = NCB * CBQ;            // Q (or dO) tile bytes
    static constexpr uint32_t TS = (BM / 64) * CBK;      // dS^T tile bytes
    // K/V buffers: two at head dim 64, so that the next work item's K and V load
    // while the current one finishes; one where shared memory has no room
    static constexpr int NKV = D == 64 ? 2 : 1;
    static constexpr uint32_t KVB = 2 * TK;              // one K + V buffer
    static constexpr uint32_t OFF_K = 0, OFF_V = TK, OFF_Q = NKV * KVB;
    static constexpr uint32_t OFF_DO = OFF_Q + QST * TQ;
    static constexpr uint32_t OFF_DS = OFF_DO + QST * TQ;
    static constexpr bool BULK_DQ = D == 64;             // staged TMA reduce-add of dQ
    static constexpr int NSTG = 1;                       // dQ staging tiles
    static constexpr uint32_t STG = BM * DH * 4;         // one f32 dQ staging tile
    static constexpr uint32_t OFF_STG = OFF_DS + TS;
    // head dim 256 (one Q/dO stage): this CTA's half of Q again, for dK, so that the
    // stage is free for the next step's Q and dO once dV has read it
    static constexpr bool QSHADOW = D == 256;
    // head dim 64: the drain warps, whose dQ leaves by TMA, also write the item's
    // dV rows, so the compute warps go straight on to the next item's first step
    // (elsewhere the compute warps write dV while the drain warps write dK)
    static constexpr bool DV_BY_DRAIN = D == 64;
    static constexpr uint32_t OFF_QSH = OFF_STG + (BULK_DQ ? NSTG * STG : 0);
    static constexpr uint32_t TQSH = (DH / 64) * CBQ;
    static constexpr uint32_t TILES = OFF_QSH + (QSHADOW ? TQSH : 0);
    // control block after the tiles: barriers, TMEM slot, abort flag, per-stage
    // LSE/Delta rows. The tiles need 1024-byte alignment (128-byte swizzle); the
    // dynamic shared memory base is 1024-aligned in practice, and SLACK covers
    // a base that is not wherever the budget leaves room (the kernel checks).
    static constexpr uint32_t OFF_TMEM_SLOT = 240, OFF_ABORT = 244;
    // LSE and Delta rows of a step, in slot (step % 2): with one Q/dO stage the
    // next step's rows arrive while phase B still reads this step's Delta
    static constexpr uint32_t OFF_LSE = 256;                        // [2][BM] f32, -LSE * log2(e)
    static constexpr uint32_t OFF_DLT = OFF_LSE + 2 * BM * 4;       // [2][BM] f32, -scale * Delta
    static constexpr uint32_t CTRL = OFF_DLT + 2 * BM * 4;
    static constexpr uint32_t SLACK = (TILES + CTRL + 1024 <= 232448) ? 1024 : 0;
    static constexpr uint32_t SMEM = SLACK + TILES + CTRL;
    // Roles: warps 0-7 compute (warp w: TMEM lanes 32 (w % 4).., query-row half
    // w / 4 of the step), 8-11 dQ drain and dK (head dim 64: and dV) epilogue,
    // 12 loads, 13 MMA issue and TMEM owner, 14-15 idle (they complete the fourth
    // warpgroup). Launched at 128 registers a thread; the fourth warpgroup gives
    // back down to REG_CTRL, the compute warpgroups grow to REG_COMPUTE, the
    // drain warpgroup to REG_DRAIN.
    static constexpr int THREADS = 512;
    static constexpr int W_DRAIN = 8, W_LOAD = 12, W_MMA = 13;
    static constexpr int REG_LAUNCH = 128, REG_CTRL = 80, REG_COMPUTE = 144, REG_DRAIN = 144;
    static_assert(4 * (REG_LAUNCH - REG_CTRL) >= 8 * (REG_COMPUTE - REG_LAUNCH) + 4 * (REG_DRAIN - REG_LAUNCH),
                  "register split");
    static_assert((2 * REG_COMPUTE + REG_DRAIN + REG_CTRL) * 32 <= 16384, "registers of one SM sub-partition");
    static constexpr int HALF = BM / 2;                  // query rows of one compute warp
    static constexpr uint32_t COL_S = 0;
    static constexpr uint32_t COL_DP = BM, COL_DV = COL_DP + BM, COL_DK = COL_DV + DH;
    static constexpr uint32_t COL_DQ = DQ_ALIAS ? COL_DP : COL_DK + DH;
    static constexpr uint32_t TMEM_COLS = 512;
    // P^T (bf16 pairs) of query rows [16 kk, 16 kk + 16): each compute warp
    // writes its half's P^T into the first columns of its own half of S^T
    static constexpr uint32_t col_p(int kk) {
        return COL_S + (uint32_t)((16 * kk / HALF) * HALF + 8 * (kk % (HALF / 16)));
    }
    static_assert(COL_DK + DH <= 512 && COL_DQ + (DQT ? BM : DH) <= 512, "tensor memory");
    static_assert(!DQ_ALIAS || (DQT ? BM : DH) <= BM, "dQ fits in the dP^T columns");
    static_assert(!DQT || DH == 128, "transposed dQ needs M = 128");
    static_assert(SMEM <= 232448, "shared memory");
    // barriers
    static constexpr int B_KV_FULL = 0;                  // [NKV]
    static constexpr int B_KV_EMPTY = NKV;               // [NKV]
    static constexpr int B_Q_FULL = 2 * NKV;             // [QST]
    static constexpr int B_Q_EMPTY = B_Q_FULL + QST;     // [QST]
    static constexpr int B_S_FULL = B_Q_EMPTY + QST;
    static constexpr int B_DS_EMPTY = B_S_FULL + 1;
    static constexpr int B_P_FULL = B_DS_EMPTY + 1;       // P^T in TMEM (8 compute warps)
    static constexpr int B_DS_FULL = B_P_FULL + 1;        // dS^T in shared memory (8 compute warps)
    static constexpr int B_DP_FULL = B_DS_FULL + 1;
    static constexpr int B_DQ_FULL = B_DP_FULL + 1;
    static constexpr int B_DQ_FREE = B_DQ_FULL + 1;
    static constexpr int B_KDONE = B_DQ_FREE + 1;        // a work item's dK, dV complete in TMEM
    static constexpr int B_EPI_DONE = B_KDONE + 1;       // ... and read out (4 drain warps, + 8 compute
                                                          // warps unless DV_BY_DRAIN)
    static constexpr int B_QSH_FULL = B_EPI_DONE + 1;    // the Q half for dK has landed (QSHADOW)
    static constexpr int B_QSH_EMPTY = B_QSH_FULL + 1;   // ... and dK has read it
    static constexpr int NBAR = B_QSH_EMPTY + 1;
    static_assert(NBAR * 8 <= (int)OFF_TMEM_SLOT, "control block");
};

// A work item: (key tile n, batch b, KV head, head-dim half h), heaviest (n = 0)
// first. Its steps walk the query tiles m_lo .. m_lo + nm - 1 of each of the G
// heads of the group.
struct BwdItem {
    int h, bkv, b, hkv, k0, m_lo, nm, steps;
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
    int q_desc;            // step order: 0 = head by head, query tiles ascending;
                           // 1 = query tiles descending from T - 1, every head per tile
};

// An item's steps in order: (query head g of the group, query tile m). Head by head,
// each CTA sweeps its own range of query tiles, so concurrent CTAs touch
// different Q, dO and dq-accumulator tiles. Descending with the heads innermost,
// the CTAs of a group that start together stay on the same query tile (every
// range ends at T - 1), so those tiles are fetched from DRAM about once and
// reused from L2 (measured on the 4K GQA layer: DRAM 1064 -> 705 MB a launch,
// 0.686 -> 0.652 ms); it was slower where the operands already fit in L2 or
// the ranges are short (windows, T = 512), and at head dim 256 and 16K.
struct BwdStep {
    int g, m;
    __device__ __forceinline__ BwdStep(const BwdItem &I, int q_desc) : g(0), m(q_desc ? I.m_lo + I.nm - 1 : I.m_lo) {}
    __device__ __forceinline__ void next(const BwdItem &I, int G, int q_desc) {
        if (q_desc) {
            if (++g == G) {
                g = 0;
                m--;
            }
        } else if (++m == I.m_lo + I.nm) {
            m = I.m_lo;
            g++;
        }
    }
};

// Epilogue of a work item: columns [c_lo, c_hi) of this thread's TMEM lane (one
// key row of dK or dV, f32, from TMEM address `taddr`) as bf16 to `row`; the
// stores are skipped for a row past the sequence end
__device__ __forceinline__ void bwd_row_out(uint32_t taddr, __nv_bfloat16 *row, int c_lo, int c_hi, bool valid) {
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(taddr + (uint32_t)c0, o);
        tmem_ld_wait(o);
        uint32_t w16[16];
#pragma unroll
        for (int e = 0; e < 16; e++) w16[e] = pack_bf16x2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1]));
        if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(row + c0);
#pragma unroll
            for (int e = 0; e < 4; e++) dst[e] = make_uint4(w16[4 * e], w16[4 * e + 1], w16[4 * e + 2], w16[4 * e + 3]);
        }
    }
}

// f32 reduction into global memory with an L2 cache-policy hint
__device__ __forceinline__ void red_add_f32_hint(float *addr, float v, uint64_t policy) {
    asm volatile("red.global.add.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(addr), "f"(v), "l"(policy) : "memory");
}

// The two phases of one key row's P / dS work (this thread's TMEM lane), 32
// query columns at a time:
//   phase A (needs S^T): P = exp2(s * scale * log2(e) - LSE * log2(e)), masked
//            to 0, as bf16 pairs pk (P^T for dV += P^T dO), and the factor g of
//            dS = g * (dP - Delta): g = P, or P (1 - tanh^2) under the cap
//            (the cap differentiated exactly: src/nn/attention.h commit log, Wave 2);
//   phase B (needs dP^T): dS = g * (dP * scale - Delta * scale) as bf16 pairs.
//   nl, nd: -LSE*log2(e) and -scale*Delta of the 32 columns (shared memory).
// CAP and MASK are compile-time so each unrolled loop is one basic block; the
// common case (neither) runs on packed f32x2 arithmetic.
template <bool CAP, bool MASK>
__device__ __forceinline__ void bwd_p32(const uint32_t (&s)[32], const float *nl, const BwdParams &p, int kj, int q0,
                                        int W, uint32_t (&pk)[16], float (&g)[32]) {
    if constexpr (!CAP && !MASK) {
        const uint64_t sl2 = f2_make(p.scale_log2, p.scale_log2);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
            const float4 a = *reinterpret_cast<const float4 *>(nl + c);
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const uint64_t y2 = f2_fma(f2_make(__uint_as_float(s[c + e]), __uint_as_float(s[c + e + 1])), sl2,
                                           e ? f2_make(a.z, a.w) : f2_make(a.x, a.y));
                float y0, y1;
                f2_split(y2, y0, y1);
                // one pair in eight of the exponentials on the FMA pipe
                const bool emu = ((c + e) & 14) == 14;
                g[c + e] = emu ? exp2_poly(y0) : ex2_approx(y0);
                g[c + e + 1] = emu ? exp2_poly(y1) : ex2_approx(y1);
                pk[(c + e) >> 1] = pack_bf16x2(g[c + e], g[c + e + 1]);
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < 32; c++) {
            const float x = __uint_as_float(s[c]);
            float pr, gg;
            const bool emu = !MASK && (c & 6) == 6;
            if constexpr (CAP) {
                const float t = tanh_via_ex2(x * p.cap_in);
                const float y = fmaf(p.cap_out, t, nl[c]);
                pr = emu ? exp2_poly(y) : ex2_approx(y);
                gg = pr * (1.0f - t * t);
            } else {
                const float y = fmaf(x, p.scale_log2, nl[c]);
                pr = emu ? exp2_poly(y) : ex2_approx(y);
                gg = pr;
            }
            if constexpr (MASK) {
                const int qi = q0 + c;
                const bool vis = kj <= qi && (W == 0 || kj > qi - W);
                pr = vis ? pr : 0.0f;
                gg = vis ? gg : 0.0f;
            }
            g[c] = gg;
            if (c & 1) pk[c >> 1] = pack_bf16x2(__uint_as_float(pk[c >> 1]), pr);
            else pk[c >> 1] = __float_as_uint(pr);
        }
    }
}

__device__ __forceinline__ void bwd_ds32(const uint32_t (&dp)[32], const float (&g)[32], const float *nd,
                                         const BwdParams &p, uint32_t (&dk)[16]) {
    const uint64_t sc2 = f2_make(p.scale, p.scale);
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
        const float4 d4 = *reinterpret_cast<const float4 *>(nd + c);
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
            const uint64_t t2 = f2_fma(f2_make(__uint_as_float(dp[c + e]), __uint_as_float(dp[c + e + 1])), sc2,
                                       e ? f2_make(d4.z, d4.w) : f2_make(d4.x, d4.y));
            float d0, d1;
            f2_split(f2_mul(f2_make(g[c + e], g[c + e + 1]), t2), d0, d1);
            dk[(c + e) >> 1] = pack_bf16x2(d0, d1);
        }
    }
}

// dS^T pairs of 32 query columns (starting at column c0 of the step) into the
// swizzled shared-memory tile: row kr, 16-byte chunk index XOR row % 8.
template <int D>
__device__ __forceinline__ void bwd_store_ds(const uint32_t (&dk)[16], int c0, int kr, uint32_t sdS) {
    using C = BwdTc<D>;
    const uint32_t blk = sdS + (uint32_t)(c0 >> 6) * C::CBK + (uint32_t)kr * 128u;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const uint32_t chunk = (uint32_t)(((c0 & 63) >> 3) + e);
        st_shared_v4(blk + ((chunk ^ (uint32_t)(kr & 7)) << 4), dk[4 * e], dk[4 * e + 1], dk[4 * e + 2],
                     dk[4 * e + 3]);
    }
}

// The MMA issuer's products, operands passed by value (shared-memory addresses
// of the operand tiles, TMEM address of the accumulator).
// S^T = K Q^T (or dP^T = V dO^T) over the full head dim.
template <class C>
__device__ __forceinline__ void bwd_mma_kq(uint32_t d_tmem, uint32_t sA, uint32_t sB) {
    constexpr uint32_t ID = idesc_bf16_f32(128, C::BM, false, false);
    const uint64_t da = sdesc_sw128(opaque_u32(sA), 16, 1024), db = sdesc_sw128(opaque_u32(sB), 16, 1024);
#pragma unroll
    for (int kk = 0; kk < C::D / 16; kk++) {
        const uint32_t oa = (kk >> 2) * C::CBK + (kk & 3) * 32;
        const uint32_t ob = (kk >> 2) * C::CBQ + (kk & 3) * 32;
        mma_ss(d_tmem, sdesc_step(da, oa), sdesc_step(db, ob), ID, kk > 0);
    }
}
// dV += P^T dO (A = P^T from TMEM; dO MN-major from the half's column blocks)
template <class C>
__device__ __forceinline__ void bwd_mma_dv(uint32_t tmem, uint32_t sdO_h, bool first) {
    constexpr uint32_t ID = idesc_bf16_f32(128, C::DH, false, true);
    const uint64_t db = sdesc_sw128(opaque_u32(sdO_h), C::CBQ, 1024);
#pragma unroll
    for (int kk = 0; kk < C::BM / 16; kk++)
        mma_ts(tmem + C::COL_DV, tmem + C::col_p(kk), sdesc_step(db, kk * 2048), ID,
               (!first || kk > 0) ? 1u : 0u);
}
// dK += dS^T Q (A = dS^T from shared memory; Q MN-major from the half's column blocks)
template <class C>
__device__ __forceinline__ void bwd_mma_dk(uint32_t tmem, uint32_t sdS, uint32_t sQ_h, bool first) {
    constexpr uint32_t ID = idesc_bf16_f32(128, C::DH, false, true);
    const uint64_t da = sdesc_sw128(opaque_u32(sdS), 16, 1024), db = sdesc_sw128(opaque_u32(sQ_h), C::CBQ, 1024);
#pragma unroll
    for (int kk = 0; kk < C::BM / 16; kk++) {
        const uint32_t oa = (kk >> 2) * C::CBK + (kk & 3) * 32;
        mma_ss(tmem + C::COL_DK, sdesc_step(da, oa), sdesc_step(db, kk * 2048), ID,
               (!first || kk > 0) ? 1u : 0u);
    }
}
// dQ = dS K, or its transpose K^T dS^T (K's half from the column blocks at sK_h)
template <class C>
__device__ __forceinline__ void bwd_mma_dq(uint32_t tmem, uint32_t sdS, uint32_t sK, uint32_t sK_h) {
    constexpr uint32_t ID =
        C::DQT ? idesc_bf16_f32(128, C::BM, true, true) : idesc_bf16_f32(128, C::D, true, true);
    const uint64_t ds_mn = sdesc_sw128(opaque_u32(sdS), C::CBK, 1024);
    const uint64_t dk_mn = sdesc_sw128(opaque_u32(C::DQT ? sK_h : sK), C::CBK, 1024);
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; kk++) {
        if constexpr (C::DQT) {
            mma_ss(tmem + C::COL_DQ, sdesc_step(dk_mn, kk * 2048), sdesc_step(ds_mn, kk * 2048), ID, kk > 0);
        } else {
            mma_ss(tmem + C::COL_DQ, sdesc_step(ds_mn, kk * 2048), sdesc_step(dk_mn, kk * 2048), ID, kk > 0);
        }
    }
}

template <class C, class P>
__device__ __forceinline__ BwdItem bwd_item(int w, const P &p) {
    BwdItem it;
    const int per_n = p.B * p.Hkv * C::NSPLIT;
    const int n = w / per_n;
    const int rest = w % per_n;
    it.h = rest % C::NSPLIT;
    it.bkv = rest / C::NSPLIT;  // b * Hkv + hkv
    it.b = it.bkv / p.Hkv;
    it.hkv = it.bkv % p.Hkv;
    it.k0 = n * C::BN;
    it.m_lo = it.k0 / C::BM;
    const int q_last = p.window > 0 ? min(p.T - 1, it.k0 + C::BN - 1 + p.window - 1) : p.T - 1;
    it.nm = q_last / C::BM - it.m_lo + 1;
    it.steps = (p.Hq / p.Hkv) * it.nm;
    return it;
}

// Persistent: gridDim.x CTAs walk the work items in the snake order above. Every
// barrier's phase counts steps (or items) over the CTA's whole run, so the
// pipeline carries on from one item into the next; TMEM is allocated once.
template <int D>
__global__ void __launch_bounds__(512, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmAcc, const BwdParams p) {
    using C = BwdTc<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const uint32_t tiles = (sbase + 1023u) & ~1023u;
    const uint32_t ctrl = tiles + C::TILES;
    uint8_t *const ctrl_p = smem_raw + (ctrl - sbase);
    const uint32_t sK0 = tiles + C::OFF_K, sQ0 = tiles + C::OFF_Q;
    const uint32_t sdO0 = tiles + C::OFF_DO, sdS = tiles + C::OFF_DS, sStg = tiles + C::OFF_STG;
    const uint32_t sQsh = tiles + C::OFF_QSH;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl_p + C::OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctrl_p + C::OFF_TMEM_SLOT);
    float *sLSE = reinterpret_cast<float *>(ctrl_p + C::OFF_LSE);
    float *sDLT = reinterpret_cast<float *>(ctrl_p + C::OFF_DLT);
    auto bar = [&](int i) -> uint32_t { return ctrl + 8u * (uint32_t)i; };
    if (tiles - sbase > C::SLACK) {
        // the layout does not fit this shared-memory base: nothing is touched
        if (threadIdx.x == 0) record_status(kStatusUnsupported);
        return;
    }

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nitems = p.num_kt * p.B * p.Hkv * C::NSPLIT;
    const int G = p.Hq / p.Hkv;
    const int W = p.window;
    auto item_of = [&](int pass) -> int { return snake_item(pass, (int)blockIdx.x, (int)gridDim.x); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NKV; s++) {
            mbar_init(bar(C::B_KV_FULL + s), 1);
            mbar_init(bar(C::B_KV_EMPTY + s), 1);
        }
        for (int s = 0; s < C::QST; s++) {
            mbar_init(bar(C::B_Q_FULL + s), 33);
            mbar_init(bar(C::B_Q_EMPTY + s), 1);
        }
        mbar_init(bar(C::B_S_FULL), 1);
        mbar_init(bar(C::B_DS_EMPTY), 1);
        mbar_init(bar(C::B_P_FULL), 8);
        mbar_init(bar(C::B_DS_FULL), 8);
        mbar_init(bar(C::B_DP_FULL), 1);
        mbar_init(bar(C::B_DQ_FULL), 1);
        mbar_init(bar(C::B_DQ_FREE), 4);
        mbar_init(bar(C::B_KDONE), 1);
        mbar_init(bar(C::B_EPI_DONE), C::DV_BY_DRAIN ? 4 : 12);
        mbar_init(bar(C::B_QSH_FULL), 1);
        mbar_init(bar(C::B_QSH_EMPTY), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::W_LOAD && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmAcc);
    }
    if (warp == C::W_MMA) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();  // the previous kernel's outputs (lse, Delta, the zeroed accumulator) are visible

    if (warp >= C::W_LOAD) {
        setmaxnreg_dec<C::REG_CTRL>();
        if (warp == C::W_LOAD) {
            // -------------------------------------------------------- producer
            int issued = 0, kv_issued = 0, qsh_issued = 0;  // loads issued (for the abort drain)
            bool ok = true;
            int gs = 0;  // step count over all of this CTA's items
            for (int pass = 0; ok; pass++) {
                const int w = item_of(pass);
                if (w >= nitems) break;
                const BwdItem I = bwd_item<C>(w, p);
                // this CTA's last item: the next kernel may start launching
                if (lane == 0 && item_of(pass + 1) >= nitems) griddep_launch_dependents();
                // K, V of the item into buffer pass % NKV once the item that used it
                // NKV items ago has no product left reading it
                const int kvs = pass % C::NKV;
                if (!mbar_wait_warp(bar(C::B_KV_EMPTY + kvs), (uint32_t)(((pass / C::NKV) & 1) ^ 1), abort_flag)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t sK = sK0 + (uint32_t)kvs * C::KVB, sV = sK + C::TK;
                    mbar_arrive_expect_tx(bar(C::B_KV_FULL + kvs), 2 * C::TK);
                    for (int c = 0; c < C::NCB; c++) {
                        tma_load_3d(sK + c * C::CBK, &tmK, bar(C::B_KV_FULL + kvs), c * 64, I.k0, I.bkv);
                        tma_load_3d(sV + c * C::CBK, &tmV, bar(C::B_KV_FULL + kvs), c * 64, I.k0, I.bkv);
                    }
                }
                kv_issued++;
                BwdStep sp(I, p.q_desc);
                for (int i = 0; i < I.steps; i++, gs++, sp.next(I, G, p.q_desc)) {
                    const int st = gs % C::QST;
                    const uint32_t ph = (uint32_t)((gs / C::QST) & 1);
                    const int g = sp.g, m = sp.m;
                    const int bhq = I.b * p.Hq + I.hkv * G + g;
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
                            tma_load_3d(sQ0 + st * C::TQ + c * C::CBQ, &tmQ, bar(C::B_Q_FULL + st), c * 64,
                                        m * C::BM, bhq);
                            tma_load_3d(sdO0 + st * C::TQ + c * C::CBQ, &tmdO, bar(C::B_Q_FULL + st), c * 64,
                                        m * C::BM, bhq);
                        }
                    }
                    issued++;
#pragma unroll
                    for (int r = 0; r < C::BM / 32; r++) {
                        sLSE[(gs & 1) * C::BM + lane + 32 * r] = -lv[r];
                        sDLT[(gs & 1) * C::BM + lane + 32 * r] = -dv[r];
                    }
                    mbar_arrive(bar(C::B_Q_FULL + st));
                    if constexpr (C::QSHADOW) {
                        // this CTA's half of Q(gs) again, for dK(gs), once dK(gs - 1) has
                        // read the previous one
                        if (!mbar_wait_warp(bar(C::B_QSH_EMPTY), (uint32_t)(gs & 1) ^ 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bar(C::B_QSH_FULL), C::TQSH);
                            for (int c = 0; c < C::DH / 64; c++)
                                tma_load_3d(sQsh + c * C::CBQ, &tmQ, bar(C::B_QSH_FULL), (I.h * (C::DH / 64) + c) * 64,
                                            m * C::BM, bhq);
                        }
                        qsh_issued++;
                    }
                }
            }
            if (!ok && lane == 0) {
                // let the copies already issued land before the CTA exits
                for (int back = 1; back <= min(kv_issued, C::NKV); back++) {
                    const int L = kv_issued - back;
                    mbar_wait_drain(bar(C::B_KV_FULL + L % C::NKV), (uint32_t)((L / C::NKV) & 1), 200000000ull);
                }
                for (int back = 1; back <= min(issued, C::QST); back++) {
                    const int L = issued - back;
                    mbar_wait_drain(bar(C::B_Q_FULL + L % C::QST), (uint32_t)((L / C::QST) & 1), 200000000ull);
                }
                if (C::QSHADOW && qsh_issued > 0)
                    mbar_wait_drain(bar(C::B_QSH_FULL), (uint32_t)((qsh_issued - 1) & 1), 200000000ull);
            }
        } else if (warp == C::W_MMA && lane == 0) {
            // ------------------------------------------------------ MMA issuer
            // S^T(j) = K Q(j)^T once stage j % QST holds Q(j) (j counts steps over all items)
            auto wait_q = [&](int j) -> bool {
                if (!mbar_wait(bar(C::B_Q_FULL + j % C::QST), (uint32_t)((j / C::QST) & 1), abort_flag)) return false;
                tc_fence_after();
                return true;
            };
            constexpr bool EARLY_S = C::QST > 1;   // S^T(j + 1) issued before dS(j) is formed
            bool ok = true;
            int gs = 0, pass = 0;
            for (; ok; pass++) {
                const int w = item_of(pass);
                if (w >= nitems) break;
                const BwdItem I = bwd_item<C>(w, p);
                const int kvs = pass % C::NKV;
                const uint32_t sK = sK0 + (uint32_t)kvs * C::KVB, sV = sK + C::TK;
                const uint32_t h_q = (uint32_t)I.h * (C::DH / 64) * C::CBQ;  // column-block offset of half h
                const uint32_t h_k = (uint32_t)I.h * (C::DH / 64) * C::CBK;
                if (!(ok = mbar_wait(bar(C::B_KV_FULL + kvs), (uint32_t)((pass / C::NKV) & 1), abort_flag))) break;
                tc_fence_after();
                if (!(ok = wait_q(gs))) break;
                bwd_mma_kq<C>(tmem + C::COL_S, sK, sQ0 + (gs % C::QST) * C::TQ);
                tc_commit(bar(C::B_S_FULL));
                // in the aliased layout dP^T overwrites the previous dQ^T: wait for its drain
                if (C::DQ_ALIAS && gs > 0) {
                    if (!(ok = mbar_wait(bar(C::B_DQ_FREE), (uint32_t)((gs - 1) & 1), abort_flag))) break;
                    tc_fence_after();
                }
                bwd_mma_kq<C>(tmem + C::COL_DP, sV, sdO0 + (gs % C::QST) * C::TQ);
                tc_commit(bar(C::B_DP_FULL));
                for (int i = 0; i < I.steps; i++, gs++) {
                    const int st = gs % C::QST;
                    const uint32_t sQ = sQ0 + st * C::TQ, sdO = sdO0 + st * C::TQ;
                    const bool more = i + 1 < I.steps;
                    // dV += P^T dO, P^T from TMEM (phase A of step gs)
                    if (!(ok = mbar_wait(bar(C::B_P_FULL), (uint32_t)(gs & 1), abort_flag))) break;
                    tc_fence_after();
                    // the first dV and dK of an item overwrite the accumulators: the
                    // previous item's must have been read out
                    if (i == 0 && pass > 0) {
                        if (!(ok = mbar_wait(bar(C::B_EPI_DONE), (uint32_t)((pass - 1) & 1), abort_flag))) break;
                        tc_fence_after();
                    }
                    bwd_mma_dv<C>(tmem, sdO + h_q, i == 0);
                    // with the Q shadow, dV(gs) is the stage's last reader
                    if constexpr (C::QSHADOW) tc_commit(bar(C::B_Q_EMPTY + st));
                    // S^T(gs + 1) over S^T(gs) / P^T(gs): phase A has read S^T(gs), and
                    // dV(gs) is ahead of it on the tensor cores. It runs while the compute
                    // warps form dS of step gs. With a single Q/dO stage Q(gs + 1) can
                    // only be loaded once dK(gs) has read Q(gs), so S^T(gs + 1) then comes
                    // after dQ(gs).
                    if (EARLY_S && more) {
                        if (!(ok = wait_q(gs + 1))) break;
                        bwd_mma_kq<C>(tmem + C::COL_S, sK, sQ0 + ((gs + 1) % C::QST) * C::TQ);
                        tc_commit(bar(C::B_S_FULL));
                    }
                    // dK += dS^T Q, then dQ (phase B of step gs). dK goes first: Q(gs + 2)
                    // (or, with one stage, Q(gs + 1)) can be loaded once the products that
                    // read Q(gs) have completed. (Issuing dQ first, so that its copy-out
                    // overlaps dK, measured slower: 0.76 against 0.68 ms on the 4K GQA
                    // layer.)
                    if (!(ok = mbar_wait(bar(C::B_DS_FULL), (uint32_t)(gs & 1), abort_flag))) break;
                    tc_fence_after();
                    if constexpr (C::QSHADOW) {
                        if (!(ok = mbar_wait(bar(C::B_QSH_FULL), (uint32_t)(gs & 1), abort_flag))) break;
                        tc_fence_after();
                        bwd_mma_dk<C>(tmem, sdS, sQsh, i == 0);
                        tc_commit(bar(C::B_QSH_EMPTY));
                    } else {
                        bwd_mma_dk<C>(tmem, sdS, sQ + h_q, i == 0);
                        tc_commit(bar(C::B_Q_EMPTY + st));  // Q, dO of this step read by every product issued
                    }
                    // the drain warps must have emptied the previous dQ (in the aliased
                    // layout they did so before dP^T(gs) was issued)
                    if (!C::DQ_ALIAS && gs > 0) {
                        if (!(ok = mbar_wait(bar(C::B_DQ_FREE), (uint32_t)((gs - 1) & 1), abort_flag))) break;
                        tc_fence_after();
                    }
                    bwd_mma_dq<C>(tmem, sdS, sK, sK + h_k);
                    tc_commit(bar(C::B_DQ_FULL));
                    tc_commit(bar(C::B_DS_EMPTY));
                    if (!EARLY_S && more) {
                        if (!(ok = wait_q(gs + 1))) break;
                        bwd_mma_kq<C>(tmem + C::COL_S, sK, sQ0 + ((gs + 1) % C::QST) * C::TQ);
                        tc_commit(bar(C::B_S_FULL));
                    }
                    if (more) {
                        // dP^T(gs + 1): phase B has read dP^T(gs); in the aliased layout it
                        // also overwrites dQ^T(gs), so wait for the drain warps
                        if (C::DQ_ALIAS) {
                            if (!(ok = mbar_wait(bar(C::B_DQ_FREE), (uint32_t)(gs & 1), abort_flag))) break;
                            tc_fence_after();
                        }
                        bwd_mma_kq<C>(tmem + C::COL_DP, sV, sdO0 + ((gs + 1) % C::QST) * C::TQ);
                        tc_commit(bar(C::B_DP_FULL));
                    }
                }
                if (!ok) break;
                tc_commit(bar(C::B_KV_EMPTY + kvs));  // K, V of this item read by every product issued
                tc_commit(bar(C::B_KDONE));           // dK, dV of this item final
            }
            if (!ok) {
                // let every product issued finish before TMEM is released
                tc_commit(bar(C::B_KDONE));
                mbar_wait_drain(bar(C::B_KDONE), (uint32_t)(pass & 1), 200000000ull);
            }
        }
    } else if (warp < C::W_DRAIN) {
        setmaxnreg_inc<C::REG_COMPUTE>();
        // ------------------------------- compute (key rows = TMEM lanes, row halves)
        const int hc = warp / 4;             // query-row half of the step
        const int kr = (warp % 4) * 32 + lane;  // key row within the tile
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const bool cap = p.softcap > 0.0f;
        bool ok = true;
        int gs = 0;
        for (int pass = 0; ok; pass++) {
            const int w = item_of(pass);
            if (w >= nitems) break;
            const BwdItem I = bwd_item<C>(w, p);
            const int kj = I.k0 + kr;
            BwdStep sp(I, p.q_desc);
            for (int i = 0; i < I.steps; i++, gs++, sp.next(I, G, p.q_desc)) {
                const int st = gs % C::QST;
                const int m = sp.m;
                const int qb = m * C::BM;
                // phase A: S^T -> P^T (TMEM) and the dS factors g (registers)
                if (!(ok = mbar_wait_warp(bar(C::B_Q_FULL + st), (uint32_t)((gs / C::QST) & 1), abort_flag))) break;
                if (!(ok = mbar_wait_warp(bar(C::B_S_FULL), (uint32_t)(gs & 1), abort_flag))) break;
                tc_fence_after();
                const float *nls = sLSE + (gs & 1) * C::BM;
                const float *nds = sDLT + (gs & 1) * C::BM;
                const bool mask = (I.k0 + C::BN - 1 > qb) || (W > 0 && I.k0 <= qb + C::BM - 1 - W);
                float g[C::HALF / 32][32];
#pragma unroll
                for (int c = 0; c < C::HALF / 32; c++) {
                    const int c0 = hc * C::HALF + 32 * c;
                    uint32_t sc[32], pk[16];
                    tmem_ld32(tmem + lane_base + C::COL_S + c0, sc);
                    tmem_ld_wait(sc);
                    if (cap) {
                        if (mask) bwd_p32<true, true>(sc, nls + c0, p, kj, qb + c0, W, pk, g[c]);
                        else bwd_p32<true, false>(sc, nls + c0, p, kj, qb + c0, W, pk, g[c]);
                    } else {
                        if (mask) bwd_p32<false, true>(sc, nls + c0, p, kj, qb + c0, W, pk, g[c]);
                        else bwd_p32<false, false>(sc, nls + c0, p, kj, qb + c0, W, pk, g[c]);
                    }
                    tmem_st16(tmem + lane_base + C::COL_S + hc * C::HALF + 16 * c, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_P_FULL));
                // phase B: dP^T -> dS^T (shared memory); the dS^T tile was last read
                // by the dK/dQ products of the previous step
                if (!(ok = mbar_wait_warp(bar(C::B_DP_FULL), (uint32_t)(gs & 1), abort_flag))) break;
                if (gs > 0 && !(ok = mbar_wait_warp(bar(C::B_DS_EMPTY), (uint32_t)((gs - 1) & 1), abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < C::HALF / 32; c++) {
                    const int c0 = hc * C::HALF + 32 * c;
                    uint32_t dc[32], dk[16];
                    tmem_ld32(tmem + lane_base + C::COL_DP + c0, dc);
                    tmem_ld_wait(dc);
                    bwd_ds32(dc, g[c], nds + c0, p, dk);
                    bwd_store_ds<D>(dk, c0, kr, sdS);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_DS_FULL));
            }
            if (!ok) break;
            if constexpr (!C::DV_BY_DRAIN) {
                // epilogue of the item: dV rows, this warp's half of the columns
                if (!(ok = mbar_wait_warp(bar(C::B_KDONE), (uint32_t)(pass & 1), abort_flag))) break;
                tc_fence_after();
                __nv_bfloat16 *row = p.dv + ((size_t)I.bkv * p.T + (size_t)min(kj, p.T - 1)) * D + I.h * C::DH;
                bwd_row_out(tmem + lane_base + C::COL_DV, row, hc * (C::DH / 2), (hc + 1) * (C::DH / 2), kj < p.T);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_EPI_DONE));
            }
        }
    } else {
        setmaxnreg_inc<C::REG_DRAIN>();
        // -------------------------------- dQ drain (warps 8..11), dK (and dV) epilogue
        const int t = threadIdx.x - 32 * C::W_DRAIN;  // TMEM lane of this thread
        const uint32_t lane_base = (uint32_t)((warp - C::W_DRAIN) * 32) << 16;
        bool ok = true;
        int gs = 0;
        for (int pass = 0; ok; pass++) {
            const int w = item_of(pass);
            if (w >= nitems) break;
            const BwdItem I = bwd_item<C>(w, p);
            BwdStep sp(I, p.q_desc);
            for (int i = 0; i < I.steps; i++, gs++, sp.next(I, G, p.q_desc)) {
                const int g = sp.g, m = sp.m;
                const int bhq = I.b * p.Hq + I.hkv * G + g;
                if (!(ok = mbar_wait_warp(bar(C::B_DQ_FULL), (uint32_t)(gs & 1), abort_flag))) break;
                tc_fence_after();
                // this thread's dQ values: a query row's DH columns, or (transposed)
                // a head-dim column's BM rows, in 32-column TMEM loads
                constexpr int NQC = (C::DQT ? C::BM : C::DH) / 32;
                uint32_t v[NQC][32];
#pragma unroll
                for (int j = 0; j < NQC; j++) tmem_ld32(tmem + lane_base + C::COL_DQ + 32 * j, v[j]);
#pragma unroll
                for (int j = 0; j < NQC; j++) tmem_ld_wait(v[j]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_DQ_FREE));
                if constexpr (C::BULK_DQ) {
                    static_assert(!C::BULK_DQ || NQC == 2, "staging covers 64 dQ values a thread");
                    const uint32_t(&v0)[32] = v[0];
                    const uint32_t(&v1)[32] = v[1 % NQC];
                    // Staging tile [BM rows][DH cols] f32, stored as DH/32 column blocks of
                    // [BM][32] with the 128-byte swizzle (16-byte chunk ^ row % 8), the
                    // layout of a TMA box {32, BM, 1}. The tile is reused once the reduce
                    // that last read it (NSTG steps ago) has read its source.
                    const uint32_t stg = sStg + (uint32_t)(gs % C::NSTG) * C::STG;
                    if (t == 0) bulk_wait_read<C::NSTG - 1>();
                    named_barrier_sync(1, 128);
                    // thread t = query row t; v = the 64 head-dim values of that row
                    const uint32_t row = stg + (uint32_t)t * 128u;
#pragma unroll
                    for (int c4 = 0; c4 < 8; c4++) {
                        const uint32_t sw = (((uint32_t)c4 ^ ((uint32_t)t & 7u)) << 4);
                        st_shared_v4(row + sw, v0[4 * c4], v0[4 * c4 + 1], v0[4 * c4 + 2], v0[4 * c4 + 3]);
                        st_shared_v4(row + (uint32_t)(C::BM * 128) + sw, v1[4 * c4], v1[4 * c4 + 1], v1[4 * c4 + 2],
                                     v1[4 * c4 + 3]);
                    }
                    fence_proxy_async_smem();
                    named_barrier_sync(1, 128);
                    if (t == 0) {
#pragma unroll
                        for (int cb = 0; cb < C::DH / 32; cb++)
                            tma_reduce_add_3d(&tmAcc, stg + (uint32_t)cb * (uint32_t)(C::BM * 128), I.h * C::DH + 32 * cb,
                                              m * C::BM, bhq);
                        bulk_commit();
                    }
                } else {
                    // lane = head-dim column h*DH + t, BM query rows: each warp-wide
                    // reduction covers 32 consecutive floats of one dQ row
                    static_assert(C::BULK_DQ || C::DQT, "per-element reduction expects the transposed dQ");

                    // evict-last: the accumulator lines are reduced into again by the
                    // other key tiles' CTAs soon, and read by the finalize
                    float *base = p.dq_acc + ((size_t)bhq * p.Tpad + (size_t)m * C::BM) * D + I.h * C::DH + t;
                    const uint64_t keep = policy_evict_last();
#pragma unroll
                    for (int j = 0; j < NQC; j++) {
#pragma unroll
                        for (int c = 0; c < 32; c++) red_add_f32_hint(base + (size_t)(32 * j + c) * D, __uint_as_float(v[j][c]), keep);
                    }
                }
            }
            if (!ok) break;
            // epilogue of the item: dK rows (and dV rows where the drain warps take them)
            if (!(ok = mbar_wait_warp(bar(C::B_KDONE), (uint32_t)(pass & 1), abort_flag))) break;
            tc_fence_after();
            const int kj = I.k0 + t;
            const size_t roff = ((size_t)I.bkv * p.T + (size_t)min(kj, p.T - 1)) * D + I.h * C::DH;
            bwd_row_out(tmem + lane_base + C::COL_DK, p.dk + roff, 0, C::DH, kj < p.T);
            if constexpr (C::DV_BY_DRAIN) bwd_row_out(tmem + lane_base + C::COL_DV, p.dv + roff, 0, C::DH, kj < p.T);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_EPI_DONE));
        }
        if constexpr (C::BULK_DQ) {
            if (t == 0) bulk_wait<0>();  // reductions complete before the CTA retires
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
