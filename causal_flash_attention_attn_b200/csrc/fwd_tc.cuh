// fwd_tc.cuh -- tensor-core forward (bf16 in, f32 accumulate) for sm_100a.
//
// One CTA per (query tile of 128 rows, batch, query head), heaviest tiles
// first. Only the KV tiles a tile can see are visited: j from
// lo = (q0 - W + 1) / 128 (0 without a window) up to the diagonal tile, so the
// cost follows the window size, as in the pages' flash kernels, which skip KV
// blocks outside the window (src/nn/attention.h commit log, Wave 2).
//
// Roles (320 threads):
//   warp 8   TMA producer: Q once, then K/V tiles through an NSTAGE ring in the
//            order the MMA warp consumes them: K0 K1 | V0 K2 | V1 K3 | ...
//   warp 9   MMA issuer (one thread) and TMEM owner (512 columns):
//            S_b = Q K_j^T into S buffer b = j % 2 (128 columns each), then
//            O += P_j V_j with P read from tensor memory (it overwrites S_b).
//            Two S buffers let QK^T of tile j+1 run while tile j is in softmax.
//   warps 0-7 softmax + epilogue: warps w and w + 4 share the TMEM lanes (query
//            rows) 32 (w % 4).. and split each row's 128 scores into halves w / 4,
//            so two warps per SM sub-partition share the exponential (and tanh)
//            work; they exchange only the row max of each tile (shared memory,
//            one named barrier per pair) and add their row sums at the end.
//            s = scale*S (or cap*tanh(scale*S/cap)), masked only on tiles that
//            straddle the diagonal or the window edge; online softmax in base 2.
//            The running max is only moved when a row max exceeds it by more
//            than 8 (a factor 256), so O in TMEM is rescaled rarely; the result
//            is exact either way because l and O use the same stale max.
// Online softmax (max, sum) per row: ARCHITECTURES.md "Vague 2" item 10.
#pragma once

#include "sm100.cuh"

namespace forge {

// Block b of a grid of ntile x nhead blocks -> (tile index heaviest first, head),
// the heads taken in groups of kHeadGroup: all tiles of a group's heads before
// the next group, so the operands a head shares across its tiles (K and V in
// the forward and the dQ kernel, Q and dO in the dK/dV kernel) are read while
// still in L2.
constexpr int kHeadGroup = 8;
__device__ __forceinline__ void grouped_block(int blk, int ntile, int nhead, int &tile_from_heavy, int &head) {
    const int full = nhead / kHeadGroup;
    const int per = ntile * kHeadGroup;
    if (blk < full * per) {
        const int g = blk / per, r = blk % per;
        tile_from_heavy = r / kHeadGroup;
        head = g * kHeadGroup + r % kHeadGroup;
    } else {
        const int r = blk - full * per, gs = nhead - full * kHeadGroup;
        tile_from_heavy = r / gs;
        head = full * kHeadGroup + r % gs;
    }
}

// DK: head dim of q and k; DV: head dim of v and o (DK = DV except for the
// decompressed multi-head latent attention, 192 / 128).
template <int DK, int DV = DK>
struct FwdTc {
    static constexpr int BM = 128, BN = 128;
    // O += P V with P split into two bf16 terms, P = hi + lo (hi = bf16(P),
    // lo = bf16(P - hi)): O is then accurate to f32 before its final rounding
    // instead of carrying the 2^-9 relative error of a single bf16 P. The
    // backward's Delta = rowsum(dO * O) inherits that accuracy; at head dim 256 a
    // single-term P moves Delta by up to ~0.2 on logits in the tanh regime.
    static constexpr bool PSPLIT = (DV == 256);
    static constexpr int NCBK = DK / 64, NCBV = DV / 64;  // 64-column (128-byte) blocks
    static constexpr uint32_t CB = 128 * 128;             // bytes of one column block of a 128-row tile
    static constexpr uint32_t TILEK = NCBK * CB;          // one 128 x DK bf16 tile (Q, K)
    static constexpr uint32_t TILEV = NCBV * CB;          // one 128 x DV bf16 tile (V)
    static constexpr uint32_t SLOT = TILEK > TILEV ? TILEK : TILEV;  // a ring slot holds a K or a V tile
    static constexpr int NSTAGE = DK == 256 ? 2 : (DK == 192 ? 3 : (DK == 128 ? 4 : 6));
    static constexpr uint32_t CTRL = 1024;                // barriers, TMEM slot, abort flag
    // after the tiles: the row-max exchange of the two column halves,
    // [2 tile parities][2 halves][128 rows] f32, and the halves' row sums [2][128]
    static constexpr uint32_t XCH = 2 * 2 * 128 * 4 + 2 * 128 * 4;
    static constexpr uint32_t SMEM = CTRL + TILEK + SLOT * NSTAGE + 1024 + XCH;
    static constexpr int THREADS = 320;
    static constexpr int W_LOAD = 8, W_MMA = 9;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O = 256;
    // barrier indices
    static constexpr int B_Q = 0;
    static constexpr int B_KV_FULL = 1;
    static constexpr int B_KV_EMPTY = 1 + NSTAGE;
    static constexpr int B_S_FULL = 1 + 2 * NSTAGE;
    static constexpr int B_P_FULL = 3 + 2 * NSTAGE;
    static constexpr int B_O_READY = 5 + 2 * NSTAGE;
    static constexpr int B_O_FINAL = 6 + 2 * NSTAGE;
    static constexpr int NBAR = 7 + 2 * NSTAGE;
    static constexpr uint32_t OFF_TMEM_SLOT = 512;
    static constexpr uint32_t OFF_ABORT = 516;
    static_assert(NBAR * 8 <= 512, "control block");
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(256 + DV <= 512, "tensor memory");
};

// Row max of a 128-column tile held as 4 x 32 registers (8 independent chains).
__device__ __forceinline__ float fwd_row_max(const uint32_t (&s)[4][32]) {
    float mx[8];
#pragma unroll
    for (int j = 0; j < 8; j++) mx[j] = __uint_as_float(s[0][j]);
#pragma unroll
    for (int c = 8; c < 128; c++) mx[c & 7] = fmaxf(mx[c & 7], __uint_as_float(s[c >> 5][c & 31]));
    return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

// Exponentials, row sum and bf16 packing of one tile row.
//   CAP:    s holds scores in log2 units; otherwise raw products, y = s*sl2 - m.
//   EMU:    every fourth column pair goes through the FMA-pipe exp2 (only for
//           tiles without masked scores), the rest through MUFU ex2.
//   PSPLIT: also leaves the residuals p - bf16(p) in s for a second PV term.
// Returns the row sum of p (f32, 4 chains).
template <bool CAP, bool EMU, bool PSPLIT>
__device__ __forceinline__ float fwd_exp_tile(uint32_t (&s)[4][32], uint32_t (&pk)[2][32], float sl2, float msub) {
    float rs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int c = 0; c < 64; c++) {
        const float x0 = __uint_as_float(s[(2 * c) >> 5][(2 * c) & 31]);
        const float x1 = __uint_as_float(s[(2 * c + 1) >> 5][(2 * c + 1) & 31]);
        const float y0 = CAP ? x0 - msub : fmaf(x0, sl2, -msub);
        const float y1 = CAP ? x1 - msub : fmaf(x1, sl2, -msub);
        float p0, p1;
        if (EMU && (c & 3) == 3) {
            p0 = exp2_poly(y0);
            p1 = exp2_poly(y1);
        } else {
            p0 = ex2_approx(y0);
            p1 = ex2_approx(y1);
        }
        rs[c & 3] += p0 + p1;
        pk[c >> 5][c & 31] = pack_bf16x2(p0, p1);
        if constexpr (PSPLIT) {
            const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&pk[c >> 5][c & 31]);
            const float2 hf = __bfloat1622float2(hi);
            s[(2 * c) >> 5][(2 * c) & 31] = __float_as_uint(p0 - hf.x);
            s[(2 * c + 1) >> 5][(2 * c + 1) & 31] = __float_as_uint(p1 - hf.y);
        }
    }
    return (rs[0] + rs[1]) + (rs[2] + rs[3]);
}

// The same for one half of a tile row (64 columns held as 2 x 32 registers);
// PSPLIT residuals are left in s. Returns the half's row sum of p.
template <bool CAP, bool EMU, bool PSPLIT>
__device__ __forceinline__ float fwd_exp_half(uint32_t (&s)[2][32], uint32_t (&pk)[32], float sl2, float msub) {
    float rs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int c = 0; c < 32; c++) {
        const float x0 = __uint_as_float(s[(2 * c) >> 5][(2 * c) & 31]);
        const float x1 = __uint_as_float(s[(2 * c + 1) >> 5][(2 * c + 1) & 31]);
        const float y0 = CAP ? x0 - msub : fmaf(x0, sl2, -msub);
        const float y1 = CAP ? x1 - msub : fmaf(x1, sl2, -msub);
        float p0, p1;
        if (EMU && (c & 3) == 3) {
            p0 = exp2_poly(y0);
            p1 = exp2_poly(y1);
        } else {
            p0 = ex2_approx(y0);
            p1 = ex2_approx(y1);
        }
        rs[c & 3] += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
        if constexpr (PSPLIT) {
            const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&pk[c]);
            const float2 hf = __bfloat1622float2(hi);
            s[(2 * c) >> 5][(2 * c) & 31] = __float_as_uint(p0 - hf.x);
            s[(2 * c + 1) >> 5][(2 * c + 1) & 31] = __float_as_uint(p1 - hf.y);
        }
    }
    return (rs[0] + rs[1]) + (rs[2] + rs[3]);
}

struct FwdParams {
    __nv_bfloat16 *o;
    float *lse;
    int B, Hq, Hkv, T, window, num_qt;
    float scale_log2;  // scale * log2(e)
    float softcap;     // 0 = off
    float cap_in;      // scale / softcap
    float cap_out;     // softcap * log2(e)
    // attention sinks: per query head logit in the softmax denominator (natural
    // units; nullptr = none). ARCHITECTURES.md family table, GPT-OSS row; "Vague
    // 2" item 10: the online softmax starts from (max, sum) = (sink, 1).
    const float *sink;
    // per (batch, query head) maximum of the scores the softmax sees, the sink
    // not included (QK-Clip's monitor, "Vague 3" item 12); nullptr = not wanted.
    // Must hold -inf (or a lower bound) before the launch: kernels atomic-max it.
    float *max_logit;
};

template <int DK, int DV = DK>
__global__ void __launch_bounds__(320, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdTc<DK, DV>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const uint32_t tiles = (sbase + C::CTRL + 1023u) & ~1023u;
    const uint32_t sQ = tiles;
    const uint32_t sKV = tiles + C::TILEK;
    float *xmax = reinterpret_cast<float *>(smem_raw + (tiles - sbase) + C::TILEK + C::SLOT * C::NSTAGE);  // [2][2][128]
    float *xsum = xmax + 2 * 2 * 128;                                                                     // [2][128]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem_raw + C::OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + C::OFF_TMEM_SLOT);
    auto bar = [&](int i) -> uint32_t { return sbase + 8u * (uint32_t)i; };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    int qt_heavy, bh;
    grouped_block((int)blockIdx.x, p.num_qt, p.B * p.Hq, qt_heavy, bh);
    const int qt = p.num_qt - 1 - qt_heavy;
    const int b = bh / p.Hq, hq = bh % p.Hq;
    const int bkv = b * p.Hkv + hq / (p.Hq / p.Hkv);
    const int q0 = qt * C::BM;
    const int lo = p.window > 0 ? max(0, q0 - p.window + 1) / C::BN : 0;
    const int n = qt - lo + 1;  // KV tiles lo..qt

    if (threadIdx.x == 0) {
        mbar_init(bar(C::B_Q), 1);
        for (int s = 0; s < C::NSTAGE; s++) {
            mbar_init(bar(C::B_KV_FULL + s), 1);
            mbar_init(bar(C::B_KV_EMPTY + s), 1);
        }
        for (int s = 0; s < 2; s++) {
            mbar_init(bar(C::B_S_FULL + s), 1);
            mbar_init(bar(C::B_P_FULL + s), 8);
        }
        mbar_init(bar(C::B_O_READY), 1);
        mbar_init(bar(C::B_O_FINAL), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::W_LOAD && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
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
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();
            mbar_arrive_expect_tx(bar(C::B_Q), C::TILEK);
            for (int c = 0; c < C::NCBK; c++) tma_load_3d(sQ + c * C::CB, &tmQ, bar(C::B_Q), c * 64, q0, bh);
            int stage = 0;
            uint32_t ph = 0;
            int issued = 0;
            bool ok = true;
            auto load = [&](const CUtensorMap *m, int j) -> bool {
                if (!mbar_wait(bar(C::B_KV_EMPTY + stage), ph ^ 1u, abort_flag)) return false;
                const bool is_v = (m == &tmV);
                mbar_arrive_expect_tx(bar(C::B_KV_FULL + stage), is_v ? C::TILEV : C::TILEK);
                for (int c = 0; c < (is_v ? C::NCBV : C::NCBK); c++)
                    tma_load_3d_hint(sKV + stage * C::SLOT + c * C::CB, m, bar(C::B_KV_FULL + stage), c * 64,
                                     j * C::BN, bkv, keep);
                issued++;
                if (++stage == C::NSTAGE) {
                    stage = 0;
                    ph ^= 1u;
                }
                return true;
            };
            ok = load(&tmK, lo);
            if (ok && n > 1) ok = load(&tmK, lo + 1);
            for (int u = 0; ok && u < n; u++) {
                ok = load(&tmV, lo + u);
                if (ok && u + 2 < n) ok = load(&tmK, lo + u + 2);
            }
            if (!ok) {
                // Let the copies already issued land before the CTA exits.
                mbar_wait_drain(bar(C::B_Q), 0, 200000000ull);
                for (int back = 1; back <= min(issued, C::NSTAGE); back++) {
                    const int L = issued - back;
                    mbar_wait_drain(bar(C::B_KV_FULL + L % C::NSTAGE), (uint32_t)((L / C::NSTAGE) & 1),
                                    200000000ull);
                }
            }
        }
    } else if (warp == C::W_MMA) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_QK = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t ID_PV = idesc_bf16_f32(128, DV, false, true);
            int stage = 0;
            uint32_t ph = 0;
            auto next = [&]() {
                if (++stage == C::NSTAGE) {
                    stage = 0;
                    ph ^= 1u;
                }
            };
            auto qk = [&](int buf) -> bool {
                if (!mbar_wait(bar(C::B_KV_FULL + stage), ph, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sK = sKV + stage * C::SLOT;
                const uint32_t dS = tmem + (buf ? C::COL_S1 : C::COL_S0);
#pragma unroll
                for (int kk = 0; kk < DK / 16; kk++) {
                    const uint32_t off = (kk >> 2) * C::CB + (kk & 3) * 32;
                    mma_ss(dS, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024), ID_QK, kk > 0);
                }
                tc_commit(bar(C::B_S_FULL + buf));
                tc_commit(bar(C::B_KV_EMPTY + stage));
                next();
                return true;
            };
            auto pv = [&](int buf, bool acc) -> bool {
                if (!mbar_wait(bar(C::B_KV_FULL + stage), ph, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sV = sKV + stage * C::SLOT;
                const uint32_t aP = tmem + (buf ? C::COL_S1 : C::COL_S0);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; kk++)
                    mma_ts(tmem + C::COL_O, aP + kk * 8, sdesc_sw128(sV + kk * 2048, C::CB, 1024), ID_PV,
                           (acc || kk > 0) ? 1u : 0u);
                if constexpr (C::PSPLIT) {
                    // low parts of P live in columns [64, 128) of the same S buffer
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; kk++)
                        mma_ts(tmem + C::COL_O, aP + 64 + kk * 8, sdesc_sw128(sV + kk * 2048, C::CB, 1024), ID_PV, 1u);
                }
                tc_commit(bar(C::B_O_READY));
                tc_commit(bar(C::B_KV_EMPTY + stage));
                next();
                return true;
            };
            bool ok = mbar_wait(bar(C::B_Q), 0, abort_flag);
            if (ok) ok = qk(0);
            if (ok && n > 1) ok = qk(1);
            for (int u = 0; ok && u < n; u++) {
                const int buf = u & 1;
                ok = mbar_wait(bar(C::B_P_FULL + buf), (uint32_t)((u >> 1) & 1), abort_flag);
                if (!ok) break;
                tc_fence_after();
                ok = pv(buf, u > 0);
                if (ok && u + 2 < n) ok = qk(buf);
            }
            // Whether or not the loop finished, O_FINAL fires once every MMA
            // issued so far has completed (the softmax warps or the abort path
            // wait on it before tensor memory is released).
            tc_commit(bar(C::B_O_FINAL));
            if (!ok) mbar_wait_drain(bar(C::B_O_FINAL), 0, 200000000ull);
        }
    } else if (warp < 8) {
        // ------------------------------------- softmax (warps 0..7, two column halves)
        const int quad = warp % 4;          // TMEM lanes 32 quad .. (query rows)
        const int hf = warp / 4;            // column half of every tile
        const int row = quad * 32 + lane;
        const int qi = q0 + row;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const uint32_t pair_bar = 1 + (uint32_t)quad;  // named barrier of warps quad, quad + 4
        const int W = p.window;
        float m = p.sink ? p.sink[hq] * kLog2e : -INFINITY;
        // the sink's 1 in the sum is counted once, by half 0
        float l = (p.sink && hf == 0) ? 1.0f : 0.0f;
        float mraw = -INFINITY;  // row max of the (log2-unit) scores, the sink excluded
        bool ok = true;
        for (int u = 0; u < n; u++) {
            const int buf = u & 1;
            const int k0 = (lo + u) * C::BN + hf * 64;  // first key of this half
            if (!mbar_wait_warp(bar(C::B_S_FULL + buf), (uint32_t)((u >> 1) & 1), abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = tmem + lane_base + (buf ? C::COL_S1 : C::COL_S0);
            uint32_t s[2][32];
            tmem_ld32(tS + hf * 64, s[0]);
            tmem_ld32(tS + hf * 64 + 32, s[1]);
            tmem_ld_wait(s[0]);
            tmem_ld_wait(s[1]);
            // capped scores are turned into log2 units here; plain ones stay raw
            // (the scale is folded into the exponent's FMA, and max commutes
            // with a positive scale)
            const bool cap = p.softcap > 0.0f;
            if (cap) {
#pragma unroll
                for (int c = 0; c < 64; c++) {
                    const float x = __uint_as_float(s[c >> 5][c & 31]);
                    s[c >> 5][c & 31] = __float_as_uint(p.cap_out * tanh_via_ex2(x * p.cap_in));
                }
            }
            const int kt0 = (lo + u) * C::BN;
            const bool need_mask = (kt0 + C::BN - 1 > q0) || (W > 0 && kt0 <= q0 + C::BM - 1 - W);
            if (need_mask) {
#pragma unroll
                for (int c = 0; c < 64; c++) {
                    const int kj = k0 + c;
                    const bool vis = kj <= qi && (W == 0 || kj > qi - W);
                    if (!vis) s[c >> 5][c & 31] = __float_as_uint(-INFINITY);
                }
            }
            float mh = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; c++) mh = fmaxf(mh, __uint_as_float(s[c >> 5][c & 31]));
            // the row max over both halves: exchange through shared memory (both
            // halves have read all their scores, so P may go over S after this)
            xmax[(buf * 2 + hf) * 128 + row] = mh;
            named_barrier_sync(pair_bar, 64);
            float mx = fmaxf(mh, xmax[(buf * 2 + (hf ^ 1)) * 128 + row]);
            if (!cap) mx *= p.scale_log2;
            mraw = fmaxf(mraw, mx);
            const float m_new = (mx > m + 8.0f) ? mx : m;
            const bool moved = (m_new != m);
            const float factor = moved ? ex2_approx(m - m_new) : 1.0f;
            if (__any_sync(0xffffffffu, moved && u > 0)) {
                // rescale this half's O columns once PV of the previous tile has landed
                if (!mbar_wait_warp(bar(C::B_O_READY), (uint32_t)((u - 1) & 1), abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float f = (moved && u > 0) ? factor : 1.0f;
#pragma unroll 1
                for (int c0 = hf * (DV / 2); c0 < (hf + 1) * (DV / 2); c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + C::COL_O + c0, o);
                    tmem_ld_wait(o);
#pragma unroll
                    for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st32(tmem + lane_base + C::COL_O + c0, o);
                }
                tmem_st_wait();
            }
            m = m_new;
            const float msub = (m == -INFINITY) ? 0.0f : m;
            uint32_t pk[32];
            float rs;
            if (cap) {
                rs = need_mask ? fwd_exp_half<true, false, C::PSPLIT>(s, pk, p.scale_log2, msub)
                               : fwd_exp_half<true, true, C::PSPLIT>(s, pk, p.scale_log2, msub);
            } else {
                rs = need_mask ? fwd_exp_half<false, false, C::PSPLIT>(s, pk, p.scale_log2, msub)
                               : fwd_exp_half<false, true, C::PSPLIT>(s, pk, p.scale_log2, msub);
            }
            // P (bf16 pairs) of this half's 64 keys: columns [32 hf, 32 hf + 32) of S
            tmem_st32(tS + hf * 32, pk);
            if constexpr (C::PSPLIT) {
                // low parts in columns [64 + 32 hf, 64 + 32 hf + 32)
#pragma unroll
                for (int c = 0; c < 32; c++)
                    pk[c] = pack_bf16x2(__uint_as_float(s[(2 * c) >> 5][(2 * c) & 31]),
                                        __uint_as_float(s[(2 * c + 1) >> 5][(2 * c + 1) & 31]));
                tmem_st32(tS + 64 + hf * 32, pk);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_P_FULL + buf));
            l = l * factor + rs;
        }
        if (ok) ok = mbar_wait_warp(bar(C::B_O_FINAL), 0, abort_flag);
        if (ok) {
            tc_fence_after();
            // both halves' row sums
            xsum[hf * 128 + row] = l;
            named_barrier_sync(pair_bar, 64);
            const float lt = l + xsum[(hf ^ 1) * 128 + row];
            const float inv_l = 1.0f / lt;
            __nv_bfloat16 *orow = p.o + ((size_t)bh * p.T + (size_t)min(qi, p.T - 1)) * DV;
#pragma unroll 1
            for (int c0 = hf * (DV / 2); c0 < (hf + 1) * (DV / 2); c0 += 32) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + C::COL_O + c0, o);
                tmem_ld_wait(o);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; i++)
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
                if (qi < p.T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
                    for (int i = 0; i < 4; i++) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            if (hf == 0) {
                if (qi < p.T) p.lse[(size_t)bh * p.T + qi] = (m + __log2f(lt)) * kLn2;
                if (p.max_logit) {
                    const float r = warp_max_f32(qi < p.T ? mraw * kLn2 : -INFINITY);
                    if (lane == 0) atomic_max_f32(p.max_logit + bh, r);
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
