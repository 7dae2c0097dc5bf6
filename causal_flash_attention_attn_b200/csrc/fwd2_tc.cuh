// fwd2_tc.cuh -- tensor-core forward with two query tiles per CTA (head dims 64
// and 128; head dim 256 uses fwd_tc.cuh, whose single tile fills TMEM).
//
// Work item: a pair of consecutive 128-row query tiles A, B of one head; one
// persistent CTA per SM walks its items (snake order over the heaviest-first
// list). The CTA streams each K/V tile once for 256 query rows and runs two softmax streams
// side by side (8 softmax warps, two per SM sub-partition): while one tile's
// scores are in softmax, the tensor cores work on the other tile. Tile A sees
// KV tiles [loA, tA], tile B [loB, tB] (tB = tA + 1); both ranges are the
// causal/window ranges of their rows, so out-of-window KV tiles are never loaded
// (the pages' flash kernels skip KV blocks outside the window, which makes the
// cost follow the window size: src/nn/attention.h commit log, Wave 2).
//
// Roles (384 threads): warps 0-3 softmax of tile A, warps 4-7 softmax of tile
// B (one thread per query row / TMEM lane), warp 8 TMA producer, warp 9 MMA
// issuer and TMEM owner, warps 10-11 idle (they complete the third warpgroup,
// whose registers the softmax warpgroups take over). TMEM: S_A, S_B (128 columns each; P overwrites its S
// as bf16), O_A, O_B (D columns each).
// MMA order per KV tile j: PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1). Because
// QK_x(j+1) is committed after PV_x(j), a softmax warp that sees S_x(j+1) also
// knows O_x holds every PV up to j, so it may rescale O_x without a wait.
// Online softmax (max, sum) per row: ARCHITECTURES.md "Vague 2" item 10.
#pragma once

#include "fwd_tc.cuh"
#include "sm100.cuh"

namespace forge {

template <int D>
struct Fwd2Tc {
    static constexpr int BM = 128, BN = 128;
    static constexpr int NCB = D / 64;
    static constexpr uint32_t CB = 128 * 128;          // column block of a 128-row tile
    static constexpr uint32_t TILE = NCB * CB;         // one 128 x D bf16 tile
    // K/V ring: four tiles (K and V of two KV tiles). At head dim 64 eight were
    // slower on short sequences: the larger first burst of loads from every CTA
    // delays the first scores (T = 512: forward 38.8 against 39.3 us)
    static constexpr int NSTAGE = 4;
    // Q buffers (tiles A and B each): two at head dim 64, so that the next work
    // item's queries load while the current item runs; one at head dim 128,
    // where shared memory has no room for a second
    static constexpr int NQB = D == 64 ? 2 : 1;
    static constexpr uint32_t CTRL = 1024;
    static constexpr uint32_t SMEM = CTRL + TILE * (2 * NQB + NSTAGE) + 1024;
    // warpgroups 0, 1: softmax of tiles A, B; warpgroup 2: producer (warp 8),
    // MMA issuer (warp 9), two idle warps. Launched at 168 registers a thread
    // (three warps per SM sub-partition); warpgroup 2 gives back down to
    // REG_CTRL so the softmax warpgroups can grow to REG_SOFTMAX:
    // 4 * (168 - REG_CTRL) >= 8 * (REG_SOFTMAX - 168). The work-item loop needs
    // REG_CTRL >= 64 (72 at head dim 64) for the producer and MMA warps to run
    // without spills.
    static constexpr int THREADS = 384;
    static constexpr int REG_LAUNCH = 168, REG_CTRL = D == 64 ? 72 : 64, REG_SOFTMAX = 216;
    // one item per CTA (no work-item loop): the control warps fit in 56
    static constexpr int REG_CTRL_ONE = 56, REG_SOFTMAX_ONE = 224;
    static_assert(4 * (REG_LAUNCH - REG_CTRL_ONE) >= 8 * (REG_SOFTMAX_ONE - REG_LAUNCH), "register split");
    static_assert(4 * (REG_LAUNCH - REG_CTRL) >= 8 * (REG_SOFTMAX - REG_LAUNCH), "register split");
    static_assert((2 * REG_SOFTMAX + REG_CTRL) * 32 <= 16384, "registers of one SM sub-partition");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t col_s(int x) { return (uint32_t)(x * 128); }
    static constexpr uint32_t col_o(int x) { return (uint32_t)(256 + x * D); }
    static constexpr int B_Q_FULL = 0;                  // [NQB]
    static constexpr int B_Q_EMPTY = NQB;               // [NQB] both tiles' O stores have read the buffer
    static constexpr int B_KV_FULL = 2 * NQB;           // [NSTAGE]
    static constexpr int B_KV_EMPTY = B_KV_FULL + NSTAGE;
    static constexpr int B_S_FULL = B_KV_EMPTY + NSTAGE;  // [2]
    static constexpr int B_P_FULL = B_S_FULL + 2;         // [2]
    static constexpr int B_O_FINAL = B_P_FULL + 2;        // [2]
    static constexpr int B_O_EMPTY = B_O_FINAL + 2;       // [2] O_x read out of TMEM
    static constexpr int NBAR = B_O_EMPTY + 2;
    static constexpr uint32_t OFF_TMEM_SLOT = 512, OFF_ABORT = 516;
    static constexpr int EMU_MASK = 7;                 // pairs with (c & 7) == 7 use the FMA-pipe exp2
    static_assert(NBAR * 8 <= 512, "control block");
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(256 + 2 * D <= 512, "tensor memory");
};

// A work item of the forward: query tiles tA = 2 pr and tB = 2 pr + 1 of head bh
// (pairs heaviest first); tile A sees KV tiles [loA, tA], tile B [loB, tB].
struct Fwd2Item {
    int bh, hq, bkv, tA, tB, qA0, qB0, loA, loB, lo, hi;
    bool hasB;
};

template <class C>
__device__ __forceinline__ Fwd2Item fwd2_item(int w, const FwdParams &p) {
    Fwd2Item I;
    const int nbh = p.B * p.Hq;
    const int npairs = (p.num_qt + 1) / 2;
    const int pr = npairs - 1 - w / nbh;
    I.bh = w % nbh;
    const int b = I.bh / p.Hq;
    I.hq = I.bh % p.Hq;
    I.bkv = b * p.Hkv + I.hq / (p.Hq / p.Hkv);
    I.tA = 2 * pr;
    I.tB = 2 * pr + 1;
    I.hasB = I.tB < p.num_qt;
    I.qA0 = I.tA * C::BM;
    I.qB0 = I.tB * C::BM;
    I.loA = p.window > 0 ? max(0, I.qA0 - p.window + 1) / C::BN : 0;
    I.loB = p.window > 0 ? max(0, I.qB0 - p.window + 1) / C::BN : 0;
    I.lo = I.loA;
    I.hi = I.hasB ? I.tB : I.tA;
    return I;
}

// Row max over 128 scores with three-input maxima (4 chains).
__device__ __forceinline__ float row_max128(const uint32_t (&s)[4][32]) {
    float mx[4];
#pragma unroll
    for (int j = 0; j < 4; j++) mx[j] = fmaxf(__uint_as_float(s[0][2 * j]), __uint_as_float(s[0][2 * j + 1]));
#pragma unroll
    for (int c = 8; c < 128; c += 8) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int a = c + 2 * j;
            mx[j] = fmax3(mx[j], __uint_as_float(s[a >> 5][a & 31]), __uint_as_float(s[(a + 1) >> 5][(a + 1) & 31]));
        }
    }
    return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// Exponentials of 32 scores (columns [32*q, 32*q + 32)), their sum (added to rs)
// and bf16 packing into pk (column pairs, low half = even column).
//   CAP: s holds log2-unit scores (y = s - m); else raw products (y = s*sl2 - m).
//   EMU: pairs with (c & EMU_MASK) == EMU_MASK use the FMA-pipe exp2.
template <bool CAP, bool EMU, int EMU_MASK>
__device__ __forceinline__ void exp_chunk32(const uint32_t (&s)[32], uint64_t sl2x2, uint64_t negm2, uint64_t (&rs)[2],
                                            uint32_t (&pk)[16]) {
#pragma unroll
    for (int c = 0; c < 16; c++) {
        const uint64_t x2 = f2_make(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1]));
        const uint64_t y2 = CAP ? f2_add(x2, negm2) : f2_fma(x2, sl2x2, negm2);
        float y0, y1;
        f2_split(y2, y0, y1);
        float p0, p1;
        if (EMU && (c & EMU_MASK) == EMU_MASK) {
            p0 = exp2_poly(y0);
            p1 = exp2_poly(y1);
        } else {
            p0 = ex2_approx(y0);
            p1 = ex2_approx(y1);
        }
        rs[c & 1] = f2_add(rs[c & 1], f2_make(p0, p1));
        pk[c] = pack_bf16x2(p0, p1);
    }
}

// Persistent: gridDim.x CTAs walk the work items (pairs of query tiles of one
// head, heaviest first) in the snake order of snake_item; barrier phases count
// KV tiles (or items) over the CTA's whole run and TMEM is allocated once.
// PERSIST = false: one CTA per item (grid = number of items), compiled without
// the work-item loop.
template <int D, bool PERSIST>
__global__ void __launch_bounds__(384, 1)
    fwd2_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const FwdParams p) {
    using C = Fwd2Tc<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const uint32_t tiles = (sbase + C::CTRL + 1023u) & ~1023u;
    const uint32_t sQ0 = tiles;                          // NQB x (Q_A, Q_B)
    const uint32_t sKV = tiles + 2 * C::NQB * C::TILE;  // NSTAGE K/V tiles
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem_raw + C::OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + C::OFF_TMEM_SLOT);
    auto bar = [&](int i) -> uint32_t { return sbase + 8u * (uint32_t)i; };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int W = p.window;
    const int nitems = ((p.num_qt + 1) / 2) * p.B * p.Hq;
    auto item_of = [&](int pass) -> int {
        return PERSIST ? snake_item(pass, (int)blockIdx.x, (int)gridDim.x) : (pass == 0 ? (int)blockIdx.x : nitems);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NQB; s++) {
            mbar_init(bar(C::B_Q_FULL + s), 1);
            mbar_init(bar(C::B_Q_EMPTY + s), 2);
        }
        for (int s = 0; s < C::NSTAGE; s++) {
            mbar_init(bar(C::B_KV_FULL + s), 1);
            mbar_init(bar(C::B_KV_EMPTY + s), 1);
        }
        for (int x = 0; x < 2; x++) {
            mbar_init(bar(C::B_S_FULL + x), 1);
            mbar_init(bar(C::B_P_FULL + x), 4);
            mbar_init(bar(C::B_O_FINAL + x), 1);
            mbar_init(bar(C::B_O_EMPTY + x), 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();  // the previous kernel's writes (q, k, v, max_logit) are visible

    if (warp >= 8) {
        setmaxnreg_dec<PERSIST ? C::REG_CTRL : C::REG_CTRL_ONE>();
        if (warp == 8) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                const uint64_t keep = policy_evict_last();
                int issued = 0, q_issued = 0;  // ring slots and Q buffers loaded (for the abort drain)
                bool ok = true;
                for (int pass = 0; ok && (PERSIST || pass == 0); pass++) {
                    const int w = item_of(pass);
                    if (w >= nitems) break;
                    const Fwd2Item I = fwd2_item<C>(w, p);
                    // this CTA's last item: the next kernel may start launching
                    if (item_of(pass + 1) >= nitems) griddep_launch_dependents();
                    // the item's queries once both O stores of the item that used this
                    // buffer NQB items ago have read it
                    const int qb = pass % C::NQB;
                    if (!mbar_wait(bar(C::B_Q_EMPTY + qb), (uint32_t)(((pass / C::NQB) & 1) ^ 1), abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sQ = sQ0 + (uint32_t)qb * 2 * C::TILE;
                    mbar_arrive_expect_tx(bar(C::B_Q_FULL + qb), I.hasB ? 2 * C::TILE : C::TILE);
                    for (int c = 0; c < C::NCB; c++) {
                        tma_load_3d(sQ + c * C::CB, &tmQ, bar(C::B_Q_FULL + qb), c * 64, I.qA0, I.bh);
                        if (I.hasB) tma_load_3d(sQ + C::TILE + c * C::CB, &tmQ, bar(C::B_Q_FULL + qb), c * 64, I.qB0, I.bh);
                    }
                    q_issued++;
                    // ring slots in order K(lo), V(lo), K(lo+1), V(lo+1), ...
                    for (int j = I.lo; ok && j <= I.hi; j++) {
                        for (int kv = 0; kv < 2 && ok; kv++) {
                            const int st = issued % C::NSTAGE;
                            const uint32_t ph = (uint32_t)((issued / C::NSTAGE) & 1);
                            if (!mbar_wait(bar(C::B_KV_EMPTY + st), ph ^ 1u, abort_flag)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(bar(C::B_KV_FULL + st), C::TILE);
                            for (int c = 0; c < C::NCB; c++)
                                tma_load_3d_hint(sKV + st * C::TILE + c * C::CB, kv ? &tmV : &tmK,
                                                 bar(C::B_KV_FULL + st), c * 64, j * C::BN, I.bkv, keep);
                            issued++;
                        }
                    }
                }
                if (!ok) {
                    for (int back = 1; back <= min(q_issued, C::NQB); back++) {
                        const int L = q_issued - back;
                        mbar_wait_drain(bar(C::B_Q_FULL + L % C::NQB), (uint32_t)((L / C::NQB) & 1), 200000000ull);
                    }
                    for (int back = 1; back <= min(issued, C::NSTAGE); back++) {
                        const int L = issued - back;
                        mbar_wait_drain(bar(C::B_KV_FULL + L % C::NSTAGE), (uint32_t)((L / C::NSTAGE) & 1), 200000000ull);
                    }
                }
            }
        } else if (warp == 9) {
            // ---------------------------------------------------------- MMA issuer
            if (lane == 0) {
                constexpr uint32_t ID_QK = idesc_bf16_f32(128, 128, false, false);
                constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, false, true);
                auto wait_full = [&](int slot) -> bool {
                    return mbar_wait(bar(C::B_KV_FULL + slot % C::NSTAGE), (uint32_t)((slot / C::NSTAGE) & 1), abort_flag);
                };
                auto release = [&](int slot) { tc_commit(bar(C::B_KV_EMPTY + slot % C::NSTAGE)); };
                int slot0 = 0;          // ring slot of the current item's K(lo)
                int cnt0 = 0, cnt1 = 0;  // PVs issued per tile over the whole run (P_FULL phases)
                bool ok = true;
                int pass = 0;
                for (; ok && (PERSIST || pass == 0); pass++) {
                    const int w = item_of(pass);
                    if (w >= nitems) break;
                    const Fwd2Item I = fwd2_item<C>(w, p);
                    const int qb = pass % C::NQB;
                    const uint32_t sQ = sQ0 + (uint32_t)qb * 2 * C::TILE;
                    // KV range of each tile ([lo_x, hi_x]; empty for a missing tile B)
                    const int lo0 = I.loA, hi0 = I.tA, lo1 = I.loB, hi1 = I.hasB ? I.tB : -1;
                    auto issue_qk = [&](int x, int slot) {
                        const uint64_t dq = sdesc_sw128(opaque_u32(sQ + (uint32_t)x * C::TILE), 16, 1024);
                        const uint64_t dk = sdesc_sw128(opaque_u32(sKV + (slot % C::NSTAGE) * C::TILE), 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < D / 16; kk++) {
                            const uint32_t off = (kk >> 2) * C::CB + (kk & 3) * 32;
                            mma_ss(tmem + C::col_s(x), sdesc_step(dq, off), sdesc_step(dk, off), ID_QK, kk > 0);
                        }
                        tc_commit(bar(C::B_S_FULL + x));
                    };
                    auto issue_pv = [&](int x, int slot, bool acc) {
                        const uint64_t dv = sdesc_sw128(opaque_u32(sKV + (slot % C::NSTAGE) * C::TILE), C::CB, 1024);
#pragma unroll
                        for (int kk = 0; kk < C::BN / 16; kk++)
                            mma_ts(tmem + C::col_o(x), tmem + C::col_s(x) + kk * 8, sdesc_step(dv, kk * 2048), ID_PV,
                                   (acc || kk > 0) ? 1u : 0u);
                    };
                    if (!(ok = mbar_wait(bar(C::B_Q_FULL + qb), (uint32_t)((pass / C::NQB) & 1), abort_flag))) break;
                    if (!(ok = wait_full(slot0))) break;
                    tc_fence_after();
                    if (I.lo >= lo0 && I.lo <= hi0) issue_qk(0, slot0);
                    if (I.lo >= lo1 && I.lo <= hi1) issue_qk(1, slot0);
                    release(slot0);
                    bool first0 = true, first1 = true;
                    for (int j = I.lo; ok && j <= I.hi; j++) {
                        const int slotV = slot0 + 2 * (j - I.lo) + 1, slotK = slotV + 1;
                        if (!(ok = wait_full(slotV))) break;
                        bool k_ready = false;
#pragma unroll
                        for (int x = 0; x < 2; x++) {
                            const int lox = x ? lo1 : lo0, hix = x ? hi1 : hi0;
                            bool &first = x ? first1 : first0;
                            int &cx = x ? cnt1 : cnt0;
                            if (ok && j >= lox && j <= hix) {
                                if (!(ok = mbar_wait(bar(C::B_P_FULL + x), (uint32_t)(cx & 1), abort_flag))) break;
                                tc_fence_after();
                                // the first PV of an item overwrites O_x: the previous
                                // item's O_x must have been read out
                                if (first && pass > 0) {
                                    if (!(ok = mbar_wait(bar(C::B_O_EMPTY + x), (uint32_t)((pass - 1) & 1), abort_flag)))
                                        break;
                                    tc_fence_after();
                                }
                                issue_pv(x, slotV, !first);
                                first = false;
                                cx++;
                            }
                            if (ok && j < I.hi && j + 1 >= lox && j + 1 <= hix) {
                                if (!k_ready) {
                                    if (!(ok = wait_full(slotK))) break;
                                    tc_fence_after();
                                    k_ready = true;
                                }
                                issue_qk(x, slotK);
                            }
                        }
                        if (!ok) break;
                        release(slotV);
                        if (j < I.hi) release(slotK);
                    }
                    if (!ok) break;
                    slot0 += 2 * (I.hi - I.lo + 1);
                    // O_FINAL fires once every MMA of the item (and before) has completed
                    tc_commit(bar(C::B_O_FINAL + 0));
                    tc_commit(bar(C::B_O_FINAL + 1));
                }
                if (!ok) {
                    tc_commit(bar(C::B_O_FINAL + 0));
                    mbar_wait_drain(bar(C::B_O_FINAL + 0), (uint32_t)(pass & 1), 200000000ull);
                }
            }
        }
    } else {
        setmaxnreg_inc<PERSIST ? C::REG_SOFTMAX : C::REG_SOFTMAX_ONE>();
        // ---------------------------------------- softmax: warps 0-3 tile A, 4-7 tile B
        const int x = warp / 4;
        const int row = threadIdx.x % 128;
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const uint32_t tS = tmem + lane_base + C::col_s(x);
        const uint32_t tO = tmem + lane_base + C::col_o(x);
        const bool cap = p.softcap > 0.0f;
        const uint64_t sl2x2 = f2_make(p.scale_log2, p.scale_log2);
        int cnt = 0;  // KV tiles of this tile slot over the whole run (S_FULL phases)
        bool ok = true;
        for (int pass = 0; ok && (PERSIST || pass == 0); pass++) {
            const int w = item_of(pass);
            if (w >= nitems) break;
            const Fwd2Item I = fwd2_item<C>(w, p);
            const int qb = pass % C::NQB;
            const bool has = (x == 0) || I.hasB;
            const int q0 = x ? I.qB0 : I.qA0;
            const int lox = x ? I.loB : I.loA, hix = x ? I.tB : I.tA;
            const int qi = q0 + row;
            const int r0 = q0 + 32 * (warp % 4);
            float m = p.sink ? p.sink[I.hq] * kLog2e : -INFINITY, l = p.sink ? 1.0f : 0.0f;
            float mraw = -INFINITY;  // row max of the (log2-unit) scores, the sink excluded
            for (int j = lox; has && j <= hix; j++, cnt++) {
                const int k0 = j * C::BN;
                if (!(ok = mbar_wait_warp(bar(C::B_S_FULL + x), (uint32_t)(cnt & 1), abort_flag))) break;
                tc_fence_after();
                uint32_t s[4][32];
                tmem_ld128x4(tS, s[0], s[1], s[2], s[3]);
                tmem_ld_wait128x4(s[0], s[1], s[2], s[3]);
                if (cap) {
#pragma unroll
                    for (int c = 0; c < 128; c++) {
                        const float v = __uint_as_float(s[c >> 5][c & 31]);
                        s[c >> 5][c & 31] = __float_as_uint(p.cap_out * tanh_via_ex2(v * p.cap_in));
                    }
                }
                // Classes of the four 32-key chunks for this warp's 32 rows
                // [r0, r0 + 31] (warp-uniform): bit q of `dead` = no key of chunk q
                // is visible to any of the rows, bit q of `part` = some are.
                unsigned dead = 0, part = 0;
#pragma unroll
                for (int q4 = 0; q4 < 4; q4++) {
                    const int c0 = k0 + 32 * q4;
                    const bool all_vis = (c0 + 31 <= r0) && (W == 0 || c0 > r0 + 31 - W);
                    const bool none = (c0 > r0 + 31) || (W > 0 && c0 + 31 <= r0 - W);
                    dead |= (unsigned)none << q4;
                    part |= (unsigned)(!all_vis && !none) << q4;
                }
                if (dead | part) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; q4++) {
                        // bit c of vm: key k0 + 32 q4 + c is visible to row qi,
                        // i.e. lo_c < c <= hi_c
                        const int hi_c = qi - (k0 + 32 * q4);
                        uint32_t vm = hi_c < 0 ? 0u : (hi_c >= 31 ? ~0u : (~0u >> (31 - hi_c)));
                        if (W > 0) {
                            const int lo_c = hi_c - W;
                            vm &= lo_c < 0 ? ~0u : (lo_c >= 31 ? 0u : (~0u << (lo_c + 1)));
                        }
#pragma unroll
                        for (int c = 0; c < 32; c++)
                            if (!((vm >> c) & 1u)) s[q4][c] = __float_as_uint(-INFINITY);
                    }
                }
                float mx = row_max128(s);
                if (!cap) mx *= p.scale_log2;
                mraw = fmaxf(mraw, mx);
                const float m_new = (mx > m + 8.0f) ? mx : m;
                const bool moved = (m_new != m);
                const float factor = moved ? ex2_approx(m - m_new) : 1.0f;
                const bool later = j > lox;  // O_x holds PVs of this item
                if (__any_sync(0xffffffffu, moved && later)) {
                    // O_x already holds every PV of this tile's earlier KV tiles
                    const float f = (moved && later) ? factor : 1.0f;
                    const uint64_t f2 = f2_make(f, f);
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld32(tO + c0, o);
                        tmem_ld_wait(o);
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            float a, bb;
                            f2_split(f2_mul(f2_make(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), f2), a, bb);
                            o[i] = __float_as_uint(a);
                            o[i + 1] = __float_as_uint(bb);
                        }
                        tmem_st32(tO + c0, o);
                    }
                }
                m = m_new;
                const float msub = (m == -INFINITY) ? 0.0f : m;
                const uint64_t negm2 = f2_make(-msub, -msub);
                uint64_t rs[2] = {f2_make(0.0f, 0.0f), f2_make(0.0f, 0.0f)};
                // 32 scores -> 16 packed P columns; P column c holds scores 2c, 2c+1.
                // Masked scores are -inf and need the MUFU exp2 (the FMA-pipe one
                // is only valid for finite arguments); chunks no row sees are 0.
                if (dead | part) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; q4++) {
                        uint32_t pk[16];
                        if ((dead >> q4) & 1u) {
#pragma unroll
                            for (int c = 0; c < 16; c++) pk[c] = 0u;
                        } else if (cap) {
                            exp_chunk32<true, false, C::EMU_MASK>(s[q4], sl2x2, negm2, rs, pk);
                        } else {
                            exp_chunk32<false, false, C::EMU_MASK>(s[q4], sl2x2, negm2, rs, pk);
                        }
                        tmem_st16(tS + 16 * q4, pk);
                    }
                } else if (cap) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; q4++) {
                        uint32_t pk[16];
                        exp_chunk32<true, true, C::EMU_MASK>(s[q4], sl2x2, negm2, rs, pk);
                        tmem_st16(tS + 16 * q4, pk);
                    }
                } else {
#pragma unroll
                    for (int q4 = 0; q4 < 4; q4++) {
                        uint32_t pk[16];
                        exp_chunk32<false, true, C::EMU_MASK>(s[q4], sl2x2, negm2, rs, pk);
                        tmem_st16(tS + 16 * q4, pk);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_P_FULL + x));
                float r0_, r1, r2, r3;
                f2_split(rs[0], r0_, r1);
                f2_split(rs[1], r2, r3);
                l = l * factor + ((r0_ + r1) + (r2 + r3));
            }
            if (!ok) break;
            if (!(ok = mbar_wait_warp(bar(C::B_O_FINAL + x), (uint32_t)(pass & 1), abort_flag))) break;
            tc_fence_after();
            // Stage this tile's O (bf16) in its Q buffer, which every MMA of the
            // item has finished reading once O_FINAL fired, in the 128-byte-swizzled
            // layout of the O tensor map, then store it with TMA (rows >= T are
            // clipped by the map).
            const uint32_t sO = sQ0 + (uint32_t)qb * 2 * C::TILE + (uint32_t)x * C::TILE;
            if (has) {
                const float inv_l = 1.0f / l;
                const uint64_t inv2 = f2_make(inv_l, inv_l);
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tO + c0, o);
                    tmem_ld_wait(o);
                    uint32_t w16[16];
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        float a, bb;
                        f2_split(f2_mul(f2_make(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), inv2), a, bb);
                        w16[i] = pack_bf16x2(a, bb);
                    }
                    const uint32_t rowaddr = sO + (uint32_t)(c0 / 64) * C::CB + (uint32_t)row * 128u;
                    const uint32_t ch0 = (uint32_t)((c0 % 64) / 8);
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        st_shared_v4(rowaddr + ((((ch0 + i) ^ (uint32_t)(row & 7))) << 4), w16[4 * i], w16[4 * i + 1],
                                     w16[4 * i + 2], w16[4 * i + 3]);
                }
            }
            // O_x is in registers / shared memory: the next item's PVs may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_O_EMPTY + x));
            if (has) {
                fence_proxy_async_smem();
                named_barrier_sync(1 + x, 128);
                if (row == 0) {
                    for (int cb = 0; cb < C::NCB; cb++) tma_store_3d(&tmO, sO + cb * C::CB, cb * 64, q0, I.bh);
                    bulk_commit();
                    bulk_wait_read<0>();
                }
                if (qi < p.T) p.lse[(size_t)I.bh * p.T + qi] = (m + __log2f(l)) * kLn2;
                if (p.max_logit) {
                    const float r = warp_max_f32(qi < p.T ? mraw * kLn2 : -INFINITY);
                    if (lane == 0) atomic_max_f32(p.max_logit + I.bh, r);
                }
            }
            // the Q buffer is free for the item NQB ahead once both tiles' stores read it
            if (row == 0) mbar_arrive(bar(C::B_Q_EMPTY + qb));
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
