// api.cu -- the C ABI of libforge_attn.so (declared in include/forge_attn.h):
// argument validation, TMA tensor maps, workspace layout and kernel dispatch.
// Single translation unit: every kernel header is included here.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "forge_attn.h"

#include "bwd_aux.cuh"
#include "bwd_dkv.cuh"
#include "bwd_tc.cuh"
#include "decode.cuh"
#include "fwd2_tc.cuh"
#include "fwd_tc.cuh"
#include "simt.cuh"
#include "sm100.cuh"

namespace forge {
namespace {

// ------------------------------------------------------------------ validation
bool aligned16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

forge_status check_sizes(int B, int Hq, int Hkv, int T, int D, forge_dtype dtype) {
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || D < 1) return FORGE_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return FORGE_ERR_INVALID_ARG;  // n_heads % n_kv_heads == 0
    if (D % 2 != 0) return FORGE_ERR_INVALID_ARG;     // head_dim even
    if (dtype != FORGE_DTYPE_F32 && dtype != FORGE_DTYPE_BF16) return FORGE_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256) return FORGE_ERR_UNSUPPORTED;
    // index arithmetic limits: grid sizes and per-tensor element counts
    const long long rows = (long long)B * Hq * T;
    if ((long long)B * Hq > (1ll << 24) || T > (1 << 30) || rows * D > (1ll << 40)) return FORGE_ERR_INVALID_ARG;
    const long long ntiles = (long long)((T + 127) / 128) * B * Hq;
    if (ntiles > 0x7fffffffll) return FORGE_ERR_INVALID_ARG;
    return FORGE_OK;
}

forge_status check_scalars(float scale, int window, float softcap) {
    if (!(scale > 0.0f) || !isfinite(scale)) return FORGE_ERR_INVALID_ARG;
    if (window < 0) return FORGE_ERR_INVALID_ARG;
    if (!(softcap >= 0.0f) || !isfinite(softcap)) return FORGE_ERR_INVALID_ARG;
    return FORGE_OK;
}

int effective_window(int window, int T) { return (window >= T) ? 0 : window; }

// Grid for kernels that take one (batch, head) pair per block row: the pairs go
// on y, and past the 65535 that y allows, on z (the kernels' `pair_index`); x
// is the kernel's own split of the rows or keys.
dim3 pair_grid(unsigned x, long long pairs) {
    const long long y = pairs < 65535 ? pairs : 65535;
    return dim3(x, (unsigned)y, (unsigned)((pairs + y - 1) / y));
}

// ------------------------------------------------------------- workspace layout
// [ delta: B*Hq*T f32, 256-aligned ][ dq accumulator: B*Hq*Tpad*D f32 (bf16 only) ]
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }
int tpad_of(int T) { return (T + 127) / 128 * 128; }
size_t delta_bytes(int B, int Hq, int T) { return round256(sizeof(float) * (size_t)B * Hq * T); }
size_t acc_bytes(int B, int Hq, int T, int D) { return round256(sizeof(float) * (size_t)B * Hq * tpad_of(T) * D); }

// Blocks of bwd_preprocess for `rows` rows of head dim D: 8 warps a block, each
// warp 32 / min(32, D / 8) rows.
unsigned preprocess_grid(long rows, int D) {
    const int lpr = D / 8 < 32 ? D / 8 : 32;
    const long per_block = 8L * (32 / lpr);
    return (unsigned)((rows + per_block - 1) / per_block);
}

// ----------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [BH][T][D] bf16 viewed as a 3D tensor (D innermost); box = 64 columns x rows x 1,
// 128-byte swizzle (the layout the tcgen05 descriptors describe). Rows past T
// read as zeros.
bool make_map(CUtensorMap *map, const void *base, int D, int T, long long BH, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * (cuuint64_t)T};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// [BH][Tpad][D] f32 accumulator as a 3D tensor; box = 32 columns (128 bytes) x
// rows x 1 with the 128-byte swizzle, the layout of the dQ staging tiles.
bool make_map_acc(CUtensorMap *map, const float *base, int D, int Tpad, long long BH, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Tpad, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)D * 4 * (cuuint64_t)Tpad};
    cuuint32_t box[3] = {32, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Text of the last CUDA error a call of this thread ran into (for diagnostics).
thread_local const char *t_last_cuda_error = "no error";

forge_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return FORGE_OK;
    t_last_cuda_error = cudaGetErrorString(e);
    return FORGE_ERR_CUDA;
}

forge_status launch_status() { return cuda_status(cudaGetLastError()); }

// SM count of the current device (cached per device), for persistent grids.
int sm_count() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// L2 size of the current device in bytes (cached per device)
long long l2_bytes() {
    static long long cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 126LL << 20;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrL2CacheSize, dev) != cudaSuccess || n < 1) n = 126 << 20;
        cache[dev] = n;
    }
    return cache[dev];
}

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel on the stream finishes (its prologue overlaps that kernel's
// tail); the kernels launched this way call griddep_wait before touching global
// memory, so the stream order of all memory effects is kept.
template <typename... KArgs, typename... Args>
forge_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                        Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...));
}

template <typename K>
forge_status set_smem(K kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return FORGE_OK;
    return cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
}

// ----------------------------------------------------------------- dispatchers
template <int D>
forge_status fwd_tc(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv, int T,
                    float scale, int window, float softcap, const float *sink, float *max_logit, cudaStream_t st) {
    using C = FwdTc<D>;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, D, T, (long long)B * Hq, 128) || !make_map(&mk, k, D, T, (long long)B * Hkv, 128) ||
        !make_map(&mv, v, D, T, (long long)B * Hkv, 128))
    {
        t_last_cuda_error = "cuTensorMapEncodeTiled failed";
        return FORGE_ERR_CUDA;
    }
    FwdParams p;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.T = T; p.window = window;
    p.num_qt = (T + 127) / 128;
    p.scale_log2 = scale * kLog2e;
    p.softcap = softcap;
    p.cap_in = softcap > 0.0f ? scale / softcap : 0.0f;
    p.cap_out = softcap * kLog2e;
    p.sink = sink;
    p.max_logit = max_logit;
    if constexpr (D == 256) {
        // one query tile per CTA: S0, S1 and the 256-column O fill TMEM
        if (set_smem(fwd_tc_kernel<D>, C::SMEM) != FORGE_OK) return FORGE_ERR_CUDA;
        const unsigned grid = (unsigned)(p.num_qt * B * Hq);
        fwd_tc_kernel<D><<<grid, C::THREADS, C::SMEM, st>>>(mq, mk, mv, p);
    } else {
        // two query tiles per CTA
        using C2 = Fwd2Tc<D>;
        CUtensorMap mo;
        if (!make_map(&mo, o, D, T, (long long)B * Hq, 128)) {
            t_last_cuda_error = "cuTensorMapEncodeTiled failed";
            return FORGE_ERR_CUDA;
        }
        if (set_smem(fwd2_tc_kernel<D, true>, C2::SMEM) != FORGE_OK ||
            set_smem(fwd2_tc_kernel<D, false>, C2::SMEM) != FORGE_OK)
            return FORGE_ERR_CUDA;
        // Persistent (one CTA per SM, the most shared memory and TMEM allow) for
        // short sequences, whose items are too light to amortise a CTA's start;
        // one CTA per item otherwise, where the hardware's dynamic placement
        // balances the uneven items better than a static order (measured forward
        // times: 16K global layer 2.57 ms persistent against 2.40 ms one CTA per
        // item; T = 512, head dim 64: 0.039 ms persistent against 0.045 ms).
        const long long items = (long long)((p.num_qt + 1) / 2) * B * Hq;
        const bool persistent = p.num_qt <= 8;
        const unsigned grid = (unsigned)(persistent && items > sm_count() ? sm_count() : items);
        // (the persistent form with grid = items takes the same items; the flag
        // only removes the work-item loop from the one-item-per-CTA code)
        if (persistent)
            return launch_pdl(fwd2_tc_kernel<D, true>, dim3(grid), dim3(C2::THREADS), C2::SMEM, st, mq, mk, mv, mo, p);
        return launch_pdl(fwd2_tc_kernel<D, false>, dim3(grid), dim3(C2::THREADS), C2::SMEM, st, mq, mk, mv, mo, p);
    }
    return launch_status();
}

// Single-tile tensor-core forward with separate key and value head dims.
template <int DK, int DV>
forge_status fwd_tc_dkv(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
                        int T, float scale, int window, float softcap, cudaStream_t st) {
    using C = FwdTc<DK, DV>;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, DK, T, (long long)B * Hq, 128) || !make_map(&mk, k, DK, T, (long long)B * Hkv, 128) ||
        !make_map(&mv, v, DV, T, (long long)B * Hkv, 128)) {
        t_last_cuda_error = "cuTensorMapEncodeTiled failed";
        return FORGE_ERR_CUDA;
    }
    FwdParams p;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.T = T; p.window = window;
    p.num_qt = (T + 127) / 128;
    p.scale_log2 = scale * kLog2e;
    p.softcap = softcap;
    p.cap_in = softcap > 0.0f ? scale / softcap : 0.0f;
    p.cap_out = softcap * kLog2e;
    p.sink = nullptr;
    p.max_logit = nullptr;
    if (set_smem(fwd_tc_kernel<DK, DV>, C::SMEM) != FORGE_OK) return FORGE_ERR_CUDA;
    fwd_tc_kernel<DK, DV><<<(unsigned)(p.num_qt * B * Hq), C::THREADS, C::SMEM, st>>>(mq, mk, mv, p);
    return launch_status();
}

template <typename T_, int DK, int DV = DK>
forge_status fwd_simt(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv, int T,
                      float scale, int window, float softcap, const float *sink, float *max_logit, cudaStream_t st) {
    const size_t sm = simt_fwd_smem<DK, DV>();
    if (set_smem(simt_fwd<T_, DK, DV>, sm) != FORGE_OK) return FORGE_ERR_CUDA;
    const dim3 grid = pair_grid((unsigned)((T + kSimtRows - 1) / kSimtRows), (long long)B * Hq);
    simt_fwd<T_, DK, DV><<<grid, kSimtThreads, sm, st>>>(static_cast<const T_ *>(q), static_cast<const T_ *>(k),
                                                     static_cast<const T_ *>(v), static_cast<T_ *>(o), lse, Hq, Hkv,
                                                     T, scale, window, softcap, sink, max_logit, B * Hq);
    return launch_status();
}

template <typename T_, int DK, int DV = DK>
forge_status bwd_simt(const void *q, const void *k, const void *v, const float *lse, const void *dO,
                      const float *delta, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int T, float scale,
                      int window, float softcap, cudaStream_t st) {
    const size_t sm1 = simt_bwd_dq_smem<DK, DV>(), sm2 = simt_bwd_dkdv_smem<DK, DV>();
    if (set_smem(simt_bwd_dq<T_, DK, DV>, sm1) != FORGE_OK || set_smem(simt_bwd_dkdv<T_, DK, DV>, sm2) != FORGE_OK)
        return FORGE_ERR_CUDA;
    const dim3 g1 = pair_grid((unsigned)((T + kSimtRows - 1) / kSimtRows), (long long)B * Hq);
    simt_bwd_dq<T_, DK, DV><<<g1, kSimtThreads, sm1, st>>>(
        static_cast<const T_ *>(q), static_cast<const T_ *>(k), static_cast<const T_ *>(v), lse,
        static_cast<const T_ *>(dO), delta, static_cast<T_ *>(dq), Hq, Hkv, T, scale, window, softcap, B * Hq);
    forge_status s = launch_status();
    if (s != FORGE_OK) return s;
    const dim3 g2 = pair_grid((unsigned)((T + kSimtRows - 1) / kSimtRows), (long long)B * Hkv);
    simt_bwd_dkdv<T_, DK, DV><<<g2, kSimtThreads, sm2, st>>>(
        static_cast<const T_ *>(q), static_cast<const T_ *>(k), static_cast<const T_ *>(v), lse,
        static_cast<const T_ *>(dO), delta, static_cast<T_ *>(dk), static_cast<T_ *>(dv), Hq, Hkv, T, scale, window,
        softcap, B * Hkv);
    return launch_status();
}

template <int D>
forge_status bwd_tc(const void *q, const void *k, const void *v, const float *lse, const void *dO,
                    const float *delta, float *acc, void *dk, void *dv, int B, int Hq, int Hkv, int T, float scale,
                    int window, float softcap, cudaStream_t st) {
    using C = BwdTc<D>;
    CUtensorMap mq, mk, mv, mdo, macc;
    if (!make_map(&mq, q, D, T, (long long)B * Hq, C::BM) || !make_map(&mk, k, D, T, (long long)B * Hkv, 128) ||
        !make_map(&mv, v, D, T, (long long)B * Hkv, 128) || !make_map(&mdo, dO, D, T, (long long)B * Hq, C::BM) ||
        !make_map_acc(&macc, acc, D, tpad_of(T), (long long)B * Hq, C::BM)) {
        t_last_cuda_error = "cuTensorMapEncodeTiled failed";
        return FORGE_ERR_CUDA;
    }
    BwdParams p;
    p.lse = lse;
    p.delta = delta;
    p.dq_acc = acc;
    p.dk = static_cast<__nv_bfloat16 *>(dk);
    p.dv = static_cast<__nv_bfloat16 *>(dv);
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.T = T; p.Tpad = tpad_of(T); p.window = window;
    p.num_kt = (T + 127) / 128;
    p.scale = scale;
    p.scale_log2 = scale * kLog2e;
    p.softcap = softcap;
    p.cap_in = softcap > 0.0f ? scale / softcap : 0.0f;
    p.cap_out = softcap * kLog2e;
    // descending query tiles where it measured faster: global causal attention at
    // head dim <= 128, T <= 8192, with Q, dO and the f32 dq accumulator larger
    // than L2 (bwd_step in bwd_tc.cuh)
    const double operand_bytes = (double)B * Hq * T * D * (2 + 2 + 4);
    p.q_desc = window == 0 && D <= 128 && T <= 8192 && operand_bytes > (double)l2_bytes() ? 1 : 0;
    if (set_smem(bwd_tc_kernel<D>, C::SMEM) != FORGE_OK) return FORGE_ERR_CUDA;
    // persistent: one CTA per SM (the kernel's shared memory and TMEM allow no
    // more), each walking its share of the work items
    const long long items = (long long)p.num_kt * B * Hkv * C::NSPLIT;
    const unsigned grid = (unsigned)(items < sm_count() ? items : sm_count());
    return launch_pdl(bwd_tc_kernel<D>, dim3(grid), dim3(C::THREADS), C::SMEM, st, mq, mk, mv, mdo, macc, p);
}

// bf16 backward with separate key and value head dims: the dK/dV kernel (one CTA
// per key tile and KV head), then the dQ kernel (one CTA per query tile and
// query head). Both read Delta from the workspace and write their outputs.
template <int DK, int DV>
forge_status bwd_tc_dkv(const void *q, const void *k, const void *v, const float *lse, const void *dO,
                        const float *delta, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int T, float scale,
                        int window, float softcap, cudaStream_t st) {
    using CA = BwdKvTc<DK, DV>;
    using CQ = BwdQTc<DK, DV>;
    CUtensorMap mq, mk, mv, mdo, mk64, mv64;
    if (!make_map(&mq, q, DK, T, (long long)B * Hq, 128) || !make_map(&mk, k, DK, T, (long long)B * Hkv, 128) ||
        !make_map(&mv, v, DV, T, (long long)B * Hkv, 128) || !make_map(&mdo, dO, DV, T, (long long)B * Hq, 128) ||
        !make_map(&mk64, k, DK, T, (long long)B * Hkv, CQ::BN) || !make_map(&mv64, v, DV, T, (long long)B * Hkv, CQ::BN)) {
        t_last_cuda_error = "cuTensorMapEncodeTiled failed";
        return FORGE_ERR_CUDA;
    }
    BwdParams p;
    p.lse = lse;
    p.delta = delta;
    p.dq_acc = nullptr;
    p.dk = static_cast<__nv_bfloat16 *>(dk);
    p.dv = static_cast<__nv_bfloat16 *>(dv);
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.T = T; p.Tpad = tpad_of(T); p.window = window;
    p.num_kt = (T + 127) / 128;
    p.scale = scale;
    p.scale_log2 = scale * kLog2e;
    p.softcap = softcap;
    p.cap_in = softcap > 0.0f ? scale / softcap : 0.0f;
    p.cap_out = softcap * kLog2e;
    p.q_desc = 0;
    if (set_smem(bwd_dkdv_tc_kernel<DK, DV>, CA::SMEM) != FORGE_OK) return FORGE_ERR_CUDA;
    bwd_dkdv_tc_kernel<DK, DV><<<(unsigned)(p.num_kt * B * Hkv), CA::THREADS, CA::SMEM, st>>>(mq, mk, mv, mdo, p);
    forge_status s = launch_status();
    if (s != FORGE_OK) return s;
    BwdQParams pq;
    pq.lse = lse;
    pq.delta = delta;
    pq.dq = static_cast<__nv_bfloat16 *>(dq);
    pq.B = B; pq.Hq = Hq; pq.Hkv = Hkv; pq.T = T; pq.window = window;
    pq.num_qt = (T + 127) / 128;
    pq.scale = p.scale; pq.scale_log2 = p.scale_log2; pq.softcap = p.softcap; pq.cap_in = p.cap_in;
    pq.cap_out = p.cap_out;
    if (set_smem(bwd_dq_tc_kernel<DK, DV>, CQ::SMEM) != FORGE_OK) return FORGE_ERR_CUDA;
    bwd_dq_tc_kernel<DK, DV><<<(unsigned)(pq.num_qt * B * Hq), CQ::THREADS, CQ::SMEM, st>>>(mq, mk64, mv64, mdo, pq);
    return launch_status();
}

// out[i] = value for i < n
__global__ void fill_f32_kernel(float *out, long n, float value) {
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = value;
}

// dsink[hq] = -sum over b, t of exp(sink[hq] - lse[b][hq][t]) * delta[b][hq][t]:
// the gradient of a per-head sink logit (its softmax column times (0 - Delta),
// the sink having no value vector). One block per query head, deterministic.
__global__ void __launch_bounds__(256) sink_grad_kernel(const float *lse, const float *delta, const float *sink,
                                                        float *dsink, int B, int Hq, int T) {
    __shared__ float part[8];
    const int hq = blockIdx.x;
    const float sg = sink[hq];
    float acc = 0.0f;
    for (long idx = threadIdx.x; idx < (long)B * T; idx += blockDim.x) {
        const long b = idx / T, t = idx % T;
        const size_t row = ((size_t)b * Hq + hq) * T + t;
        acc -= expf(sg - lse[row]) * delta[row];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        float sum = 0.0f;
        for (int w = 0; w < 8; w++) sum += part[w];
        dsink[hq] = sum;
    }
}

// Keys per decode chunk, multiples of 64: enough chunks for about 16 CTAs per SM.
// The warp-pipelined split kernel keeps six CTAs resident per SM at head dim 128,
// so this gives several waves with a short tail (measured on B 16, Hkv 8, 16K
// keys: 5.40 TB/s at 16 per SM, 5.36 at 24, 5.32 at 32, 5.03 at 8).
constexpr long kDecCtasPerSm = 16;
int decode_chunk(int B, int Hkv, int T) {
    const long per = (long)B * Hkv;
    const long splits = (kDecCtasPerSm * 148 + per - 1) / per;
    long chunk = ((T + splits - 1) / splits + 63) / 64 * 64;
    return (int)(chunk < 64 ? 64 : chunk);
}

template <typename T_, int D, int MG>
forge_status decode_split_launch(const void *q, const void *kc, const void *vc, const DecParams &p, cudaStream_t st) {
    using C = DecCfg<T_, D>;
    if (set_smem(decode_split<T_, D, MG>, C::smem(MG)) != FORGE_OK) return FORGE_ERR_CUDA;
    decode_split<T_, D, MG><<<pair_grid((unsigned)p.nsplit, (long long)p.B * p.Hkv), kDecThreads,
                              C::smem(p.Hq / p.Hkv), st>>>(static_cast<const T_ *>(q), static_cast<const T_ *>(kc),
                                                           static_cast<const T_ *>(vc), p);
    return launch_status();
}

// The warp-pipelined kernel serves groups whose queries and outputs fit a lane's
// registers (MG * D <= 1024) with steps of at most 8 KB of K rows; decode_split
// the others.
template <typename T_, int D, int MG>
constexpr bool decode_warp_fits() {
    return MG * D <= 1024 && (32 / MG) * D * (int)sizeof(T_) <= 8192;
}

template <typename T_, int D, int MG>
forge_status decode_pick(const void *q, const void *kc, const void *vc, const DecParams &p, cudaStream_t st) {
    if constexpr (decode_warp_fits<T_, D, MG>()) {
        using C = DecWCfg<T_, D, MG>;
        if (set_smem(decode_split_warp<T_, D, MG>, C::SMEM) != FORGE_OK) return FORGE_ERR_CUDA;
        decode_split_warp<T_, D, MG><<<pair_grid((unsigned)p.nsplit, (long long)p.B * p.Hkv), kDecWarps * 32, C::SMEM,
                                       st>>>(static_cast<const T_ *>(q), static_cast<const T_ *>(kc),
                                             static_cast<const T_ *>(vc), p);
        return launch_status();
    } else {
        return decode_split_launch<T_, D, (MG < 4 ? 4 : MG)>(q, kc, vc, p, st);
    }
}

template <typename T_, int D>
forge_status decode_run(const void *q, const void *kc, const void *vc, void *o, DecParams p, cudaStream_t st) {
    const int G = p.Hq / p.Hkv;
    forge_status s = G <= 1   ? decode_pick<T_, D, 1>(q, kc, vc, p, st)
                     : G <= 2 ? decode_pick<T_, D, 2>(q, kc, vc, p, st)
                     : G <= 4 ? decode_pick<T_, D, 4>(q, kc, vc, p, st)
                     : G <= 8 ? decode_pick<T_, D, 8>(q, kc, vc, p, st)
                              : decode_pick<T_, D, 16>(q, kc, vc, p, st);
    if (s != FORGE_OK) return s;
    decode_combine<T_, D><<<(unsigned)(p.B * p.Hq), D, 0, st>>>(static_cast<T_ *>(o), p);
    return launch_status();
}

#define FORGE_DISPATCH_D(D, ...)                               \
    switch (D) {                                               \
        case 64: { constexpr int kD = 64; __VA_ARGS__ } break;   \
        case 128: { constexpr int kD = 128; __VA_ARGS__ } break; \
        case 256: { constexpr int kD = 256; __VA_ARGS__ } break; \
        default: return FORGE_ERR_UNSUPPORTED;                 \
    }

}  // namespace

// Timeout self-test: waits on a barrier nothing completes.
__global__ void selftest_timeout_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t barrier;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&barrier), 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&barrier), 0, &abort_flag, limit_ns);
    __syncthreads();
}

// exp2 self-test: the kernels' FMA-pipe exp2 next to CUDA's exp2f.
__global__ void selftest_exp2_kernel(const float *x, float *y, float *y_ref, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        y[i] = exp2_poly(x[i]);
        y_ref[i] = exp2f(x[i]);
    }
}

}  // namespace forge

// ---------------------------------------------------------------------------
// Backward without caller-provided workspace.
//
// Some callers cannot allocate device memory at all: a host program that only
// receives device buffers from another runtime and has no allocator of its own
// (plain C or a foreign-language binding), or a process whose memory pool owns
// the whole device and forbids allocations outside it. forge_attn_bwd_noalloc
// serves them with scratch that lives in this fixed-size device array instead
// of a caller workspace. Every GPU that loads the library holds the array until
// the process exits. Its device address belongs to the device's current
// context: it is looked up on the first call made with that device current and
// cached together with the context's unique id, and looked up again when the
// id has changed (a cudaDeviceReset ends the old context, and the module and
// its array get a new address in the next one).
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
struct NoAllocEntry {
    unsigned long long ctx_id;  // id of the context the address belongs to
    void *ptr;
};
NoAllocEntry g_noalloc[kNoAllocMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

template <typename F>
F driver_fn(const char *name) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<F>(ptr);
    return nullptr;
}

// Unique id of the calling thread's current context (never reused within the
// process), or 0 when there is none or the driver cannot say.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (get_current == nullptr || get_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

forge_status noalloc_scratch_for_current_device(void **out) {
    int dev = -1;
    forge_status s = forge::cuda_status(cudaGetDevice(&dev));
    if (s != FORGE_OK) return s;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return FORGE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoAllocEntry &e = g_noalloc[dev];
    const unsigned long long id = current_context_id();
    if (e.ptr == nullptr || id == 0 || id != e.ctx_id) {
        // first call on this device, a context without a readable id (looked up
        // every time then), or a new context since the last lookup
        void *p = nullptr;
        s = forge::cuda_status(cudaGetSymbolAddress(&p, g_noalloc_scratch));
        if (s != FORGE_OK) return s;
        e.ptr = p;
        e.ctx_id = current_context_id();  // the lookup may have created the context
    }
    *out = e.ptr;
    return FORGE_OK;
}
}  // namespace

using namespace forge;

extern "C" {

forge_status forge_attn_fwd_ext(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                                int Hkv, int T, int D, float scale, int window, float softcap, const float *sink,
                                float *max_logit, forge_dtype dtype, void *stream) {
    forge_status s = check_sizes(B, Hq, Hkv, T, D, dtype);
    if (s != FORGE_OK) return s;
    if ((s = check_scalars(scale, window, softcap)) != FORGE_OK) return s;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FORGE_ERR_INVALID_ARG;
    if ((sink != nullptr && !aligned4(sink)) || (max_logit != nullptr && !aligned4(max_logit)))
        return FORGE_ERR_INVALID_ARG;
    window = effective_window(window, T);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (max_logit != nullptr) {
        const long n = (long)B * Hq;
        fill_f32_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(max_logit, n, -INFINITY);
        if ((s = launch_status()) != FORGE_OK) return s;
    }
    if (dtype == FORGE_DTYPE_BF16) {
        FORGE_DISPATCH_D(D, return fwd_tc<kD>(q, k, v, o, lse, B, Hq, Hkv, T, scale, window, softcap, sink,
                                               max_logit, st);)
    } else {
        FORGE_DISPATCH_D(D, return fwd_simt<float, kD>(q, k, v, o, lse, B, Hq, Hkv, T, scale, window, softcap, sink,
                                                        max_logit, st);)
    }
    return FORGE_ERR_UNSUPPORTED;
}

forge_status forge_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                            int Hkv, int T, int D, float scale, int window, float softcap, forge_dtype dtype,
                            void *stream) {
    return forge_attn_fwd_ext(q, k, v, o, lse, B, Hq, Hkv, T, D, scale, window, softcap, nullptr, nullptr, dtype,
                              stream);
}

size_t forge_attn_bwd_workspace_size(int B, int Hq, int Hkv, int T, int D, forge_dtype dtype) {
    if (check_sizes(B, Hq, Hkv, T, D, dtype) != FORGE_OK) return 0;
    size_t n = delta_bytes(B, Hq, T);
    if (dtype == FORGE_DTYPE_BF16) n += acc_bytes(B, Hq, T, D);
    return n;
}

static forge_status check_workspace(void *ws, size_t bytes, int B, int Hq, int Hkv, int T, int D, forge_dtype dtype) {
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FORGE_ERR_WORKSPACE;
    if (bytes < forge_attn_bwd_workspace_size(B, Hq, Hkv, T, D, dtype)) return FORGE_ERR_WORKSPACE;
    return FORGE_OK;
}

forge_status forge_attn_bwd_preprocess(const void *o, const void *dO, int B, int Hq, int Hkv, int T, int D,
                                       forge_dtype dtype, void *workspace, size_t workspace_bytes, void *stream) {
    forge_status s = check_sizes(B, Hq, Hkv, T, D, dtype);
    if (s != FORGE_OK) return s;
    if (!aligned16(o) || !aligned16(dO)) return FORGE_ERR_INVALID_ARG;
    if ((s = check_workspace(workspace, workspace_bytes, B, Hq, Hkv, T, D, dtype)) != FORGE_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *delta = static_cast<float *>(workspace);
    const long rows = (long)B * Hq * T;
    const unsigned grid = preprocess_grid(rows, D);
    if (dtype == FORGE_DTYPE_BF16) {
        // the dq accumulator receives reductions: zero it in the same pass
        float *acc = reinterpret_cast<float *>(static_cast<char *>(workspace) + delta_bytes(B, Hq, T));
        FORGE_DISPATCH_D(D, return launch_pdl(bwd_preprocess<__nv_bfloat16, kD>, dim3(grid), dim3(256), 0, st,
                                              static_cast<const __nv_bfloat16 *>(o),
                                              static_cast<const __nv_bfloat16 *>(dO), delta, acc, rows, T,
                                              tpad_of(T));)
    }
    FORGE_DISPATCH_D(D, return launch_pdl(bwd_preprocess<float, kD>, dim3(grid), dim3(256), 0, st,
                                          static_cast<const float *>(o), static_cast<const float *>(dO), delta,
                                          static_cast<float *>(nullptr), rows, T, tpad_of(T));)
    return FORGE_ERR_UNSUPPORTED;
}

forge_status forge_attn_bwd_main(const void *q, const void *k, const void *v, const float *lse, const void *dO,
                                 void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int T, int D, float scale,
                                 int window, float softcap, forge_dtype dtype, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    forge_status s = check_sizes(B, Hq, Hkv, T, D, dtype);
    if (s != FORGE_OK) return s;
    if ((s = check_scalars(scale, window, softcap)) != FORGE_OK) return s;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lse) || !aligned16(dO) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv))
        return FORGE_ERR_INVALID_ARG;
    if ((s = check_workspace(workspace, workspace_bytes, B, Hq, Hkv, T, D, dtype)) != FORGE_OK) return s;
    window = effective_window(window, T);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float *delta = static_cast<const float *>(workspace);
    if (dtype == FORGE_DTYPE_BF16) {
        float *acc = reinterpret_cast<float *>(static_cast<char *>(workspace) + delta_bytes(B, Hq, T));
        FORGE_DISPATCH_D(D, return bwd_tc<kD>(q, k, v, lse, dO, delta, acc, dk, dv, B, Hq, Hkv, T, scale, window,
                                              softcap, st);)
    }
    FORGE_DISPATCH_D(D, return bwd_simt<float, kD>(q, k, v, lse, dO, delta, dq, dk, dv, B, Hq, Hkv, T, scale, window,
                                                   softcap, st);)
    return FORGE_ERR_UNSUPPORTED;
}

forge_status forge_attn_bwd_finalize(void *dq, int B, int Hq, int Hkv, int T, int D, forge_dtype dtype,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    forge_status s = check_sizes(B, Hq, Hkv, T, D, dtype);
    if (s != FORGE_OK) return s;
    if (!aligned16(dq)) return FORGE_ERR_INVALID_ARG;
    if ((s = check_workspace(workspace, workspace_bytes, B, Hq, Hkv, T, D, dtype)) != FORGE_OK) return s;
    if (dtype != FORGE_DTYPE_BF16) return FORGE_OK;  // f32: dq already written by the main stage
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float *acc = reinterpret_cast<const float *>(static_cast<char *>(workspace) + delta_bytes(B, Hq, T));
    const long long total = (long long)B * Hq * T * (D / 8);
    const unsigned grid = (unsigned)((total + 255) / 256);
    FORGE_DISPATCH_D(D, return launch_pdl(bwd_finalize_dq<kD>, dim3(grid), dim3(256), 0, st, acc,
                                          static_cast<__nv_bfloat16 *>(dq), (long)B * Hq, T, tpad_of(T));)
    return FORGE_ERR_UNSUPPORTED;
}

forge_status forge_attn_bwd_ext(const void *q, const void *k, const void *v, const void *o, const float *lse,
                                const void *dO, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int T, int D,
                                float scale, int window, float softcap, const float *sink, float *dsink,
                                forge_dtype dtype, void *workspace, size_t workspace_bytes, void *stream) {
    forge_status s = check_sizes(B, Hq, Hkv, T, D, dtype);
    if (s != FORGE_OK) return s;
    if ((s = check_scalars(scale, window, softcap)) != FORGE_OK) return s;
    // validate everything before the first launch: on error nothing runs
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FORGE_ERR_INVALID_ARG;
    if (dsink != nullptr && (!aligned4(dsink) || !aligned4(sink))) return FORGE_ERR_INVALID_ARG;
    if (sink != nullptr && !aligned4(sink)) return FORGE_ERR_INVALID_ARG;
    if ((s = check_workspace(workspace, workspace_bytes, B, Hq, Hkv, T, D, dtype)) != FORGE_OK) return s;
    s = forge_attn_bwd_preprocess(o, dO, B, Hq, Hkv, T, D, dtype, workspace, workspace_bytes, stream);
    if (s != FORGE_OK) return s;
    if (dsink != nullptr) {
        // the sink enters dq, dk, dv only through lse; its own gradient needs Delta
        sink_grad_kernel<<<(unsigned)Hq, 256, 0, static_cast<cudaStream_t>(stream)>>>(
            lse, static_cast<const float *>(workspace), sink, dsink, B, Hq, T);
        if ((s = launch_status()) != FORGE_OK) return s;
    }
    s = forge_attn_bwd_main(q, k, v, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap, dtype, workspace,
                            workspace_bytes, stream);
    if (s != FORGE_OK) return s;
    return forge_attn_bwd_finalize(dq, B, Hq, Hkv, T, D, dtype, workspace, workspace_bytes, stream);
}

forge_status forge_attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                            const void *dO, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int T, int D,
                            float scale, int window, float softcap, forge_dtype dtype, void *workspace,
                            size_t workspace_bytes, void *stream) {
    return forge_attn_bwd_ext(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap, nullptr,
                              nullptr, dtype, workspace, workspace_bytes, stream);
}

forge_status forge_attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const float *lse,
                                    const void *dO, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int T, int D,
                                    float scale, int window, float softcap, forge_dtype dtype, void *stream) {
    forge_status s = check_sizes(B, Hq, Hkv, T, D, dtype);
    if (s != FORGE_OK) return s;
    if (forge_attn_bwd_workspace_size(B, Hq, Hkv, T, D, dtype) > kNoAllocScratchBytes) {
        t_last_cuda_error = "problem too large for forge_attn_bwd_noalloc's 32 MiB scratch";
        return FORGE_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    if ((s = noalloc_scratch_for_current_device(&scratch)) != FORGE_OK) return s;
    // the preprocess stage zeroes the dq accumulator rows and overwrites Delta,
    // so whatever the previous call left in the array does not matter
    return forge_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap, dtype, scratch,
                          kNoAllocScratchBytes, stream);
}

// d_k != d_v at (d_k, d_v) = (192, 128), the decompressed multi-head latent
// attention of the DeepSeek V3 family: on the tensor cores (bf16) or the CUDA
// cores (f32), forward and backward.
static bool dkv_supported(int Dk, int Dv, forge_dtype dtype) {
    return (dtype == FORGE_DTYPE_F32 || dtype == FORGE_DTYPE_BF16) && Dk == 192 && Dv == 128;
}
static bool dkv_fwd_supported(int Dk, int Dv, forge_dtype dtype) { return dkv_supported(Dk, Dv, dtype); }

size_t forge_attn_bwd_workspace_size_dkv(int B, int Hq, int Hkv, int T, int Dk, int Dv, forge_dtype dtype) {
    if (Dk == Dv) return forge_attn_bwd_workspace_size(B, Hq, Hkv, T, Dk, dtype);
    if (!dkv_supported(Dk, Dv, dtype) || check_sizes(B, Hq, Hkv, T, Dv, dtype) != FORGE_OK) return 0;
    return delta_bytes(B, Hq, T);  // Delta only: both paths write dq directly
}

forge_status forge_attn_fwd_dkv(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                                int Hkv, int T, int Dk, int Dv, float scale, int window, float softcap,
                                forge_dtype dtype, void *stream) {
    if (Dk == Dv) return forge_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, T, Dk, scale, window, softcap, dtype, stream);
    forge_status s = check_sizes(B, Hq, Hkv, T, Dv, dtype);
    if (s != FORGE_OK) return s;
    if (!dkv_fwd_supported(Dk, Dv, dtype)) return FORGE_ERR_UNSUPPORTED;
    if ((s = check_scalars(scale, window, softcap)) != FORGE_OK) return s;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FORGE_ERR_INVALID_ARG;
    window = effective_window(window, T);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == FORGE_DTYPE_BF16) return fwd_tc_dkv<192, 128>(q, k, v, o, lse, B, Hq, Hkv, T, scale, window, softcap, st);
    return fwd_simt<float, 192, 128>(q, k, v, o, lse, B, Hq, Hkv, T, scale, window, softcap, nullptr, nullptr, st);
}

forge_status forge_attn_bwd_dkv(const void *q, const void *k, const void *v, const void *o, const float *lse,
                                const void *dO, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int T, int Dk,
                                int Dv, float scale, int window, float softcap, forge_dtype dtype, void *workspace,
                                size_t workspace_bytes, void *stream) {
    if (Dk == Dv)
        return forge_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, Dk, scale, window, softcap, dtype,
                              workspace, workspace_bytes, stream);
    forge_status s = check_sizes(B, Hq, Hkv, T, Dv, dtype);
    if (s != FORGE_OK) return s;
    if (!dkv_supported(Dk, Dv, dtype)) return FORGE_ERR_UNSUPPORTED;
    if ((s = check_scalars(scale, window, softcap)) != FORGE_OK) return s;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FORGE_ERR_INVALID_ARG;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
        workspace_bytes < forge_attn_bwd_workspace_size_dkv(B, Hq, Hkv, T, Dk, Dv, dtype))
        return FORGE_ERR_WORKSPACE;
    window = effective_window(window, T);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *delta = static_cast<float *>(workspace);
    const long rows = (long)B * Hq * T;
    if (dtype == FORGE_DTYPE_BF16) {
        bwd_preprocess<__nv_bfloat16, 128><<<preprocess_grid(rows, 128), 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dO), delta, nullptr, rows, T,
            tpad_of(T));
        if ((s = launch_status()) != FORGE_OK) return s;
        return bwd_tc_dkv<192, 128>(q, k, v, lse, dO, delta, dq, dk, dv, B, Hq, Hkv, T, scale, window, softcap, st);
    }
    bwd_preprocess<float, 128><<<preprocess_grid(rows, 128), 256, 0, st>>>(
        static_cast<const float *>(o), static_cast<const float *>(dO), delta, nullptr, rows, T, tpad_of(T));
    if ((s = launch_status()) != FORGE_OK) return s;
    return bwd_simt<float, 192, 128>(q, k, v, lse, dO, delta, dq, dk, dv, B, Hq, Hkv, T, scale, window, softcap, st);
}

size_t forge_attn_decode_workspace_size(int B, int Hq, int Hkv, int T, int D) {
    if (check_sizes(B, Hq, Hkv, T, D, FORGE_DTYPE_BF16) != FORGE_OK) return 0;
    const int chunk = decode_chunk(B, Hkv, T);
    const long nsplit = (T + chunk - 1) / chunk;
    return ((size_t)B * Hq * nsplit * (size_t)(D + 2) * sizeof(float) + 255) / 256 * 256;
}

forge_status forge_attn_decode(const void *q, const void *k_cache, const void *v_cache, void *o, float *lse,
                               const int *seq_lens, int B, int Hq, int Hkv, int T, int Tmax, int D, float scale,
                               int window, float softcap, const float *sink, forge_dtype dtype, void *workspace,
                               size_t workspace_bytes, void *stream) {
    forge_status s = check_sizes(B, Hq, Hkv, T, D, dtype);
    if (s != FORGE_OK) return s;
    if ((s = check_scalars(scale, window, softcap)) != FORGE_OK) return s;
    if (Tmax < T || (long)Tmax * D * B * Hkv > (1L << 40)) return FORGE_ERR_INVALID_ARG;
    if (Hq / Hkv > kDecMaxG) return FORGE_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return FORGE_ERR_INVALID_ARG;
    if ((lse && !aligned4(lse)) || (seq_lens && !aligned4(seq_lens)) || (sink && !aligned4(sink)))
        return FORGE_ERR_INVALID_ARG;
    const size_t need = forge_attn_decode_workspace_size(B, Hq, Hkv, T, D);
    if (!aligned16(workspace) || workspace_bytes < need) return FORGE_ERR_WORKSPACE;
    DecParams p;
    p.seq_lens = seq_lens;
    p.sink = sink;
    p.part = static_cast<float *>(workspace);
    p.lse = lse;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.T = T; p.Tmax = Tmax;
    p.window = effective_window(window, T);
    p.chunk = decode_chunk(B, Hkv, T);
    p.nsplit = (T + p.chunk - 1) / p.chunk;
    p.qscale = softcap > 0.0f ? scale / softcap : scale * kLog2e;
    p.cap_out = softcap > 0.0f ? softcap * kLog2e : 0.0f;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == FORGE_DTYPE_BF16) {
        FORGE_DISPATCH_D(D, return decode_run<__nv_bfloat16, kD>(q, k_cache, v_cache, o, p, st);)
    } else {
        FORGE_DISPATCH_D(D, return decode_run<float, kD>(q, k_cache, v_cache, o, p, st);)
    }
    return FORGE_ERR_UNSUPPORTED;
}

forge_status forge_attn_check(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    forge_status s = cuda_status(cudaStreamSynchronize(st));
    if (s != FORGE_OK) return s;
    int h = 0;
    if ((s = cuda_status(cudaMemcpyFromSymbol(&h, g_status, sizeof(int)))) != FORGE_OK) return s;
    if (h != 0) {
        const int zero = 0;
        if ((s = cuda_status(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)))) != FORGE_OK) return s;
        return static_cast<forge_status>(h);
    }
    return FORGE_OK;
}

const char *forge_attn_status_string(forge_status s) {
    switch (s) {
        case FORGE_OK: return "FORGE_OK";
        case FORGE_ERR_INVALID_ARG: return "FORGE_ERR_INVALID_ARG: invalid argument";
        case FORGE_ERR_UNSUPPORTED: return "FORGE_ERR_UNSUPPORTED: unsupported configuration";
        case FORGE_ERR_WORKSPACE: return "FORGE_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case FORGE_ERR_CUDA: return "FORGE_ERR_CUDA: CUDA runtime or launch failure";
        case FORGE_ERR_TIMEOUT: return "FORGE_ERR_TIMEOUT: a bounded wait inside a kernel ran out";
    }
    return "FORGE_ERR_UNKNOWN";
}

forge_status forge_attn_selftest_timeout(unsigned int limit_us, void *stream) {
    if (limit_us < 1 || limit_us > 2000000u) return FORGE_ERR_INVALID_ARG;
    selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * limit_us);
    return launch_status();
}

forge_status forge_attn_selftest_exp2(const float *x, float *y, float *y_ref, int n, void *stream) {
    if (n < 0 || (n > 0 && (x == nullptr || y == nullptr || y_ref == nullptr))) return FORGE_ERR_INVALID_ARG;
    if (n == 0) return FORGE_OK;
    selftest_exp2_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, y_ref, n);
    return launch_status();
}

const char *forge_attn_last_cuda_error(void) { return t_last_cuda_error; }

forge_status forge_attn_timeout_info(unsigned int *info4) {
    if (info4 == nullptr) return FORGE_ERR_INVALID_ARG;
    forge_status s = cuda_status(cudaMemcpyFromSymbol(info4, g_timeout_info, 4 * sizeof(unsigned)));
    if (s != FORGE_OK) return s;
    const unsigned zero[4] = {0, 0, 0, 0};
    return cuda_status(cudaMemcpyToSymbol(g_timeout_info, zero, sizeof(zero)));
}

const char *forge_attn_version(void) { return "forge_attn 0.1.0 sm_100a"; }

}  // extern "C"
