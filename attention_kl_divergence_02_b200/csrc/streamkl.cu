// streamkl.cu -- host side of libstreamkl: argument checks, TMA descriptors and launches
// behind the C ABI declared in include/streamkl.h.  The whole library is this one
// translation unit (the kernels are headers), so the device status word has one home.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>

#include "streamkl.h"
#include "sm100.cuh"
#include "fwd_kernel.cuh"
#include "fwd_keys_kernel.cuh"
#include "bwd_kernel.cuh"
#include "watchdog.cuh"
#include "probe.cuh"

namespace {

thread_local char t_last_cuda_error[256] = "";

int cuda_fail(cudaError_t e, const char* what) {
    snprintf(t_last_cuda_error, sizeof(t_last_cuda_error), "%s: %s", what, cudaGetErrorString(e));
    return STREAMKL_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D view [planes, rows, d] of a dense bf16 tensor, box_rows-row x 64-column boxes
// (128 rows unless asked), 128-byte swizzle, zero fill outside the tensor.
int make_map(CUtensorMap* map, const void* base, long long planes, long long rows, int d,
             unsigned box_rows = 128) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        snprintf(t_last_cuda_error, sizeof(t_last_cuda_error), "cuTensorMapEncodeTiled unavailable");
        return STREAMKL_ERR_CUDA;
    }
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(t_last_cuda_error, sizeof(t_last_cuda_error), "cuTensorMapEncodeTiled failed (%d)",
                 (int)r);
        return STREAMKL_ERR_CUDA;
    }
    return STREAMKL_OK;
}

constexpr int kMaxDevices = 64;
constexpr int kDefaultSMs = 148;   // B200; used only when no device can be queried
constexpr int kKeysMaxRows = 8;    // query rows up to which the forward runs keys as MMA rows

// SM count of the current device, looked up once per device ordinal (it cannot change while
// the process runs).  The split heuristics size their grids in waves of one CTA per SM.
int num_sms() {
    static std::mutex mu;
    static int cache[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();   // no device here (host-only queries): clear and use the default
        return kDefaultSMs;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            return kDefaultSMs;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int Hq, int Hkv, int NQ, int NK, int d, float scale, int causal) {
    if (B < 1 || Hq < 1 || Hkv < 1 || NQ < 1 || NK < 1 || d < 1) return STREAMKL_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return STREAMKL_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return STREAMKL_ERR_UNSUPPORTED;
    if (Hq % Hkv != 0) return STREAMKL_ERR_UNSUPPORTED;
    if (causal && NQ != NK) return STREAMKL_ERR_UNSUPPORTED;
    if ((long long)B * Hq * NQ >= (1ll << 31) || (long long)B * Hkv * NK >= (1ll << 31))
        return STREAMKL_ERR_UNSUPPORTED;
    return STREAMKL_OK;
}

template <typename K>
int set_smem(K kernel, int bytes) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    return STREAMKL_OK;
}

template <int D, bool SHARED>
int launch_fwd(const CUtensorMap& q1, const CUtensorMap& q2, const CUtensorMap& k1,
               const CUtensorMap& k2, const skl::FwdParams& p, int grid, cudaStream_t st) {
    auto kern = p.kl21 ? skl::streamkl_fwd_kernel<D, SHARED, true> : skl::streamkl_fwd_kernel<D, SHARED, false>;
    constexpr int smem = skl::FwdCfg<D>::kSmem;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    kern<<<grid, skl::kFwdThreads, smem, st>>>(q1, q2, k1, k2, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "streamkl_fwd launch");
    return STREAMKL_OK;
}

template <int D, bool SHARED, int ROWS>
int launch_fwd_keys(const CUtensorMap& q1, const CUtensorMap& q2, const CUtensorMap& k1,
                    const CUtensorMap& k2, const skl::FwdParams& p, int grid, cudaStream_t st) {
    auto kern = p.kl21 ? skl::streamkl_fwd_keys_kernel<D, SHARED, ROWS, true>
                       : skl::streamkl_fwd_keys_kernel<D, SHARED, ROWS, false>;
    constexpr int smem = skl::KeysCfg<D>::kSmem;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    kern<<<grid, skl::kKeysThreads, smem, st>>>(q1, q2, k1, k2, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "streamkl_fwd (few rows) launch");
    return STREAMKL_OK;
}

template <int D, bool SHARED>
int launch_fwd_keys_rows(const CUtensorMap& q1, const CUtensorMap& q2, const CUtensorMap& k1,
                         const CUtensorMap& k2, const skl::FwdParams& p, int grid, cudaStream_t st) {
    return p.NQ == 1 ? launch_fwd_keys<D, SHARED, 1>(q1, q2, k1, k2, p, grid, st)
                     : launch_fwd_keys<D, SHARED, 8>(q1, q2, k1, k2, p, grid, st);
}

// fp32 tile-blocked workspace -> bf16 rows (scale applied), one launch.
template <int D>
int launch_convert(const float* ws, uint16_t* out, int planes, int rows, int ntiles, float scale,
                   cudaStream_t st, const char* what) {
    const size_t threads = (size_t)planes * ntiles * 128 * (D / 32);
    size_t blocks = (threads + 255) / 256;
    const size_t cap = (size_t)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    skl::streamkl_tile_convert_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(ws, out, planes, rows, ntiles,
                                                                          scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    return STREAMKL_OK;
}

template <int D, bool SHARED, int HP>
int launch_bwd(int mode, const CUtensorMap& q1, const CUtensorMap& q2, const CUtensorMap& k1,
               const CUtensorMap& k2, const skl::BwdParams& p, int grid, size_t ws_bytes,
               uint16_t* dk, cudaStream_t st) {
    auto kern = mode == 1 ? skl::streamkl_bwd_kernel<D, SHARED, 1, HP>
                          : skl::streamkl_bwd_kernel<D, SHARED, 2, HP>;
    constexpr int smem = skl::BwdCfg<D, SHARED, HP>::kSmem;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    cudaError_t e = cudaMemsetAsync(p.dk_ws, 0, ws_bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "workspace memset");
    kern<<<grid, skl::kBwdThreads, smem, st>>>(q1, q2, k1, k2, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "streamkl_bwd launch");
    rc = launch_convert<D>(p.dk_ws, dk, p.B * p.Hkv, p.NK, p.nkt, p.scale, st, "dk convert launch");
    if (rc || p.splits == 1) return rc;
    return launch_convert<D>(p.dq_ws, p.dq, p.B * p.Hq, p.NQ, p.nqt, p.scale, st, "dq convert launch");
}

}  // namespace

extern "C" {

int streamkl_version(void) { return 100; }

const char* streamkl_status_string(int status) {
    switch (status) {
        case STREAMKL_OK: return "ok";
        case STREAMKL_ERR_INVALID_ARG: return "invalid argument";
        case STREAMKL_ERR_UNSUPPORTED: return "unsupported shape, scale or alignment";
        case STREAMKL_ERR_CUDA: return "CUDA error";
        case STREAMKL_ERR_TIMEOUT: return "a kernel pipeline wait timed out";
        default: return "unknown status";
    }
}

const char* streamkl_last_cuda_error(void) { return t_last_cuda_error; }

int streamkl_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, skl::g_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "read device status");
    if (v != 0) {
        e = cudaMemcpyToSymbol(skl::g_status, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "clear device status");
    }
    return v;
}

int streamkl_selftest_watchdog(int starve, long long* waited_ns, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned long long zero[3] = {0, 0, 0};
    cudaError_t e = cudaMemcpyToSymbolAsync(skl::g_watchdog, zero, sizeof(zero), 0,
                                            cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "watchdog reset");
    skl::streamkl_watchdog_kernel<<<1, 64, 0, st>>>(starve);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "watchdog launch");
    const int status = streamkl_device_status(stream);   // synchronises, reads, clears
    if (status == STREAMKL_ERR_CUDA) return status;
    unsigned long long res[3];
    e = cudaMemcpyFromSymbol(res, skl::g_watchdog, sizeof(res));
    if (e != cudaSuccess) return cuda_fail(e, "watchdog read");
    if (waited_ns) {
        waited_ns[0] = (long long)res[1];
        waited_ns[1] = (long long)res[2];
    }
    // both waits must agree with the status: all passed (OK) or none did (TIMEOUT)
    if (status == STREAMKL_OK && res[0] != 3ull) return STREAMKL_ERR_TIMEOUT;
    if (status != STREAMKL_OK && res[0] != 0ull) return STREAMKL_ERR_CUDA;
    return status;
}


int streamkl_probe_exp2(int kind, int iters, long long* n_exp, void* stream) {
    if ((kind != 0 && kind != 1) || iters < 1) return STREAMKL_ERR_INVALID_ARG;
    const int grid = 4 * num_sms();
    const long long n = (long long)grid * skl::kProbeThreads * skl::kProbeChains * iters;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kind == 0)
        skl::streamkl_probe_exp2_kernel<0><<<grid, skl::kProbeThreads, 0, st>>>(iters, 0, nullptr);
    else
        skl::streamkl_probe_exp2_kernel<1><<<grid, skl::kProbeThreads, 0, st>>>(iters, 0, nullptr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "exp2 probe launch");
    if (n_exp) *n_exp = n;
    return STREAMKL_OK;
}

int streamkl_num_sms(void) { return num_sms(); }

int streamkl_eval_exp2(int kind, const float* x, float* y, long long n, void* stream) {
    if ((kind != 0 && kind != 1) || n < 0 || (n > 0 && (!x || !y))) return STREAMKL_ERR_INVALID_ARG;
    if (n == 0) return STREAMKL_OK;
    const long long blocks = std::min<long long>((n + 511) / 512, 8ll * num_sms());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kind == 0)
        skl::streamkl_eval_exp2_kernel<0><<<(unsigned)blocks, 256, 0, st>>>(x, y, n);
    else
        skl::streamkl_eval_exp2_kernel<1><<<(unsigned)blocks, 256, 0, st>>>(x, y, n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "exp2 evaluation launch");
    return STREAMKL_OK;
}

int streamkl_probe_clock(long long duration_ns, long long interval_ns, long long* samples,
                         int max_pairs, void* stream) {
    if (!samples) return STREAMKL_ERR_INVALID_ARG;
    if (duration_ns < 1000 || duration_ns > 10000000000LL || interval_ns < 1000 ||
        interval_ns > duration_ns || max_pairs < 2)
        return STREAMKL_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(samples) % 8 != 0) return STREAMKL_ERR_UNSUPPORTED;
    skl::streamkl_probe_clock_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        duration_ns, interval_ns, max_pairs, samples);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "clock probe launch");
    return STREAMKL_OK;
}

}  // extern "C"

namespace {


// Key tiles per range for `splits` ranges, and the number of non-empty ranges that gives.
void split_ranges(int NK, int splits, int* kps, int* used) {
    const int nkt = (NK + 127) / 128;
    const int s = std::max(1, std::min(splits, nkt));
    *kps = (nkt + s - 1) / s;
    *used = (nkt + *kps - 1) / *kps;
}

// The split-K merge, launched as a programmatic dependent of the forward kernel just queued on
// the same stream: its launch and ramp overlap that grid's last CTAs, and its first
// instruction waits until the forward grid has completed and its partial states are visible.
int launch_merge(const float* part, int splits, long long R, float scale, float* kl, float* lse1,
                 float* lse2, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min<long long>((R + 255) / 256, 8ll * num_sms()));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, skl::streamkl_splitk_merge_kernel, part, splits, R, scale,
                                       kl, lse1, lse2);
    if (e != cudaSuccess) return cuda_fail(e, "split-K merge launch");
    return STREAMKL_OK;
}

// kl21 != nullptr: the symmetric variant (also KL(P2 || P1) per row), one key range only.
int fwd_impl(const uint16_t* q1, const uint16_t* k1, const uint16_t* q2, const uint16_t* k2, int B,
             int Hq, int Hkv, int NQ, int NK, int d, float scale, int causal, int splits, float* kl,
             float* lse1, float* lse2, float* part, float* kl21, void* stream) {
    const bool shared = (k1 == k2);
    CUtensorMap mq1, mq2, mk1, mk2;
    int rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (NQ <= kKeysMaxRows) {
        // at most 8 query rows: keys as the MMA's rows (16-row query boxes, rows past NQ zero)
        if ((rc = make_map(&mq1, q1, (long long)B * Hq, NQ, d, 16))) return rc;
        if ((rc = make_map(&mq2, q2, (long long)B * Hq, NQ, d, 16))) return rc;
        if ((rc = make_map(&mk1, k1, (long long)B * Hkv, NK, d))) return rc;
        if ((rc = make_map(&mk2, k2, (long long)B * Hkv, NK, d))) return rc;
        skl::FwdParams p;
        p.rep4 = 0;
        p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.NQ = NQ; p.NK = NK;
        p.causal = causal ? 1 : 0;
        p.n_qblk = 1;
        p.sl2 = scale * 1.4426950408889634f;
        p.scale = scale;
        p.kl = kl; p.lse1 = lse1; p.lse2 = lse2;
        p.kl21 = kl21;
        split_ranges(NK, splits, &p.kps, &p.splits);
        p.part = p.splits > 1 ? part : nullptr;
        const long long grid = (long long)B * Hq * p.splits;
        if (grid >= (1ll << 31)) return STREAMKL_ERR_UNSUPPORTED;
        if (d == 128) {
            rc = shared ? launch_fwd_keys_rows<128, true>(mq1, mq2, mk1, mk2, p, (int)grid, st)
                        : launch_fwd_keys_rows<128, false>(mq1, mq2, mk1, mk2, p, (int)grid, st);
        } else {
            rc = shared ? launch_fwd_keys_rows<64, true>(mq1, mq2, mk1, mk2, p, (int)grid, st)
                        : launch_fwd_keys_rows<64, false>(mq1, mq2, mk1, mk2, p, (int)grid, st);
        }
        if (rc || p.splits == 1) return rc;
        return launch_merge(part, p.splits, (long long)B * Hq * NQ, scale, kl, lse1, lse2, st);
    }
    // at most 32 query rows: they are loaded once into each 32-lane quarter of the query
    // tile (32-row boxes), so that all four warps of a warpgroup can fold them
    const int rep4 = NQ <= 32 ? 1 : 0;
    if ((rc = make_map(&mq1, q1, (long long)B * Hq, NQ, d, rep4 ? 32 : 128))) return rc;
    if ((rc = make_map(&mq2, q2, (long long)B * Hq, NQ, d, rep4 ? 32 : 128))) return rc;
    if ((rc = make_map(&mk1, k1, (long long)B * Hkv, NK, d))) return rc;
    if ((rc = make_map(&mk2, k2, (long long)B * Hkv, NK, d))) return rc;
    skl::FwdParams p;
    p.rep4 = rep4;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.NQ = NQ; p.NK = NK;
    p.causal = causal ? 1 : 0;
    p.n_qblk = (NQ + 255) / 256;
    p.sl2 = scale * 1.4426950408889634f;
    p.scale = scale;
    p.kl = kl; p.lse1 = lse1; p.lse2 = lse2;
    p.kl21 = kl21;
    split_ranges(NK, splits, &p.kps, &p.splits);
    p.part = p.splits > 1 ? part : nullptr;
    const long long grid = (long long)B * Hq * p.n_qblk * p.splits;
    if (grid >= (1ll << 31)) return STREAMKL_ERR_UNSUPPORTED;
    if (d == 128) {
        rc = shared ? launch_fwd<128, true>(mq1, mq2, mk1, mk2, p, (int)grid, st)
                    : launch_fwd<128, false>(mq1, mq2, mk1, mk2, p, (int)grid, st);
    } else {
        rc = shared ? launch_fwd<64, true>(mq1, mq2, mk1, mk2, p, (int)grid, st)
                    : launch_fwd<64, false>(mq1, mq2, mk1, mk2, p, (int)grid, st);
    }
    if (rc || p.splits == 1) return rc;
    return launch_merge(part, p.splits, (long long)B * Hq * NQ, scale, kl, lse1, lse2, st);
}

}  // namespace

extern "C" {

int streamkl_fwd(const uint16_t* q1, const uint16_t* k1, const uint16_t* q2, const uint16_t* k2,
                 int B, int Hq, int Hkv, int NQ, int NK, int d, float scale, int causal,
                 float* kl, float* lse1, float* lse2, void* stream) {
    if (!q1 || !k1 || !q2 || !k2 || !kl || !lse1 || !lse2) return STREAMKL_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, NQ, NK, d, scale, causal);
    if (rc) return rc;
    if (!aligned16(q1) || !aligned16(k1) || !aligned16(q2) || !aligned16(k2) || !aligned16(kl) ||
        !aligned16(lse1) || !aligned16(lse2))
        return STREAMKL_ERR_UNSUPPORTED;
    return fwd_impl(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, 1, kl, lse1, lse2,
                    nullptr, nullptr, stream);
}

int streamkl_fwd_sym(const uint16_t* q1, const uint16_t* k1, const uint16_t* q2, const uint16_t* k2,
                     int B, int Hq, int Hkv, int NQ, int NK, int d, float scale, int causal,
                     float* kl12, float* kl21, float* lse1, float* lse2, void* stream) {
    if (!q1 || !k1 || !q2 || !k2 || !kl12 || !kl21 || !lse1 || !lse2) return STREAMKL_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, NQ, NK, d, scale, causal);
    if (rc) return rc;
    const void* ptrs[] = {q1, k1, q2, k2, kl12, kl21, lse1, lse2};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return STREAMKL_ERR_UNSUPPORTED;
    return fwd_impl(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, 1, kl12, lse1, lse2,
                    nullptr, kl21, stream);
}

int streamkl_fwd_splits(int B, int Hq, int NQ, int NK) {
    if (B < 1 || Hq < 1 || NQ < 1 || NK < 1) return 1;
    if (NQ <= kKeysMaxRows) {
        // keys as MMA rows: one wave of two CTAs per SM, every CTA streaming its key range
        const long long heads = (long long)B * Hq;
        const int nkt = (NK + 127) / 128;
        const long long want = (2ll * num_sms()) / heads;
        if (want <= 1 || nkt < 2) return 1;
        int kps, used;
        split_ranges(NK, (int)std::min<long long>(want, nkt), &kps, &used);
        return used;
    }
    const long long blocks = (long long)B * Hq * ((NQ + 255) / 256);
    const int nkt = (NK + 127) / 128;
    const int sms = num_sms();
    if (blocks >= sms || nkt < 2) return 1;
    // time model: waves of one CTA per SM, each CTA ~ its key tiles + 8 tiles of fixed cost
    // (query load, pipeline fill and drain, partial store; 8 measured on B4 H32 NQ1 NK32768,
    // where 128 blocks already fill the GPU and splitting lost 6 %); the fewest ranges within
    // 3 % of the best
    double best = 1e300;
    int best_s = 1;
    std::vector<double> cost(65, 0.0);
    for (int s = 1; s <= std::min(nkt, 64); ++s) {
        int kps, used;
        split_ranges(NK, s, &kps, &used);
        const long long ctas = blocks * used;
        const double waves = (double)((ctas + sms - 1) / sms);
        cost[s] = waves * (kps + 8);
        if (cost[s] < best) best = cost[s];
    }
    for (int s = 1; s <= std::min(nkt, 64); ++s) {
        if (cost[s] <= best * 1.03) {
            best_s = s;
            break;
        }
    }
    int kps, used;
    split_ranges(NK, best_s, &kps, &used);
    return used;
}

size_t streamkl_fwd_splitk_workspace_bytes(int B, int Hq, int NQ, int NK, int splits) {
    if (B < 1 || Hq < 1 || NQ < 1 || NK < 1 || splits < 0) return 0;
    if (splits == 0) splits = streamkl_fwd_splits(B, Hq, NQ, NK);
    int kps, used;
    split_ranges(NK, splits, &kps, &used);
    if (used <= 1) return 0;
    return (size_t)used * 5 * B * Hq * NQ * sizeof(float);
}

int streamkl_fwd_splitk(const uint16_t* q1, const uint16_t* k1, const uint16_t* q2,
                        const uint16_t* k2, int B, int Hq, int Hkv, int NQ, int NK, int d,
                        float scale, int causal, int splits, float* kl, float* lse1, float* lse2,
                        void* workspace, size_t workspace_bytes, void* stream) {
    if (!q1 || !k1 || !q2 || !k2 || !kl || !lse1 || !lse2 || splits < 0) return STREAMKL_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, NQ, NK, d, scale, causal);
    if (rc) return rc;
    if (!aligned16(q1) || !aligned16(k1) || !aligned16(q2) || !aligned16(k2) || !aligned16(kl) ||
        !aligned16(lse1) || !aligned16(lse2) || !aligned16(workspace))
        return STREAMKL_ERR_UNSUPPORTED;
    if (splits == 0) splits = streamkl_fwd_splits(B, Hq, NQ, NK);
    const size_t need = streamkl_fwd_splitk_workspace_bytes(B, Hq, NQ, NK, splits);
    if (need > 0 && (!workspace || workspace_bytes < need)) return STREAMKL_ERR_INVALID_ARG;
    return fwd_impl(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, splits, kl, lse1, lse2,
                    static_cast<float*>(workspace), nullptr, stream);
}

}  // extern "C"

namespace {

// Query heads per backward CTA: 2 at d = 64 when every KV group has an even number of query
// heads (the two heads' dK partials of a key tile then meet in tensor memory and their key
// tiles are loaded once), else 1.  At d = 128 tensor memory has no room for a second dQ.
int bwd_heads_per_cta(int Hq, int Hkv, int d) {
    return (d == 64 && (Hq / Hkv) % 2 == 0) ? 2 : 1;
}

// Key ranges per query tile for the backward: 1 when the query tiles fill the GPU, else the
// fewest ranges within 3 % of the best of a waves x (tiles per range + 6) model (6 tiles of
// fixed cost per CTA: query load, pipeline fill, dQ reduction), at most 32.
int bwd_splits(int B, int Hq, int Hkv, int NQ, int NK, int d) {
    const long long ctas = (long long)B * (Hq / bwd_heads_per_cta(Hq, Hkv, d)) * ((NQ + 127) / 128);
    const int nkt = (NK + 127) / 128;
    const int sms = num_sms();
    if (ctas >= sms || nkt < 2) return 1;
    double cost[33] = {0};
    double best = 1e300;
    for (int s = 1; s <= std::min(nkt, 32); ++s) {
        int kps, used;
        split_ranges(NK, s, &kps, &used);
        const double waves = (double)((ctas * used + sms - 1) / sms);
        cost[s] = waves * (kps + 6);
        best = std::min(best, cost[s]);
    }
    for (int s = 1; s <= std::min(nkt, 32); ++s) {
        if (cost[s] <= best * 1.03) {
            int kps, used;
            split_ranges(NK, s, &kps, &used);
            return used;
        }
    }
    return 1;
}

size_t bwd_dk_bytes(int B, int Hkv, int NK, int d) {
    const size_t rows = (size_t)(NK + 127) / 128 * 128;   // whole 128-row key tiles
    return (size_t)B * Hkv * rows * d * sizeof(float);
}

}  // namespace

extern "C" {

size_t streamkl_bwd_workspace_bytes(int B, int Hq, int Hkv, int NQ, int NK, int d) {
    if (B < 1 || Hq < 1 || Hkv < 1 || NQ < 1 || NK < 1 || (d != 64 && d != 128)) return 0;
    size_t bytes = bwd_dk_bytes(B, Hkv, NK, d);
    if (bwd_splits(B, Hq, Hkv, NQ, NK, d) > 1)   // plus the dQ partial sums, tile-blocked
        bytes += (size_t)B * Hq * ((NQ + 127) / 128 * 128) * d * sizeof(float);
    return bytes;
}

int streamkl_bwd(int mode, const uint16_t* q1, const uint16_t* k1, const uint16_t* q2,
                 const uint16_t* k2, const float* kl, const float* lse1, const float* lse2,
                 const float* dkl, int B, int Hq, int Hkv, int NQ, int NK, int d, float scale,
                 int causal, uint16_t* dq, uint16_t* dk, void* workspace, size_t workspace_bytes,
                 void* stream) {
    if (mode != 1 && mode != 2) return STREAMKL_ERR_INVALID_ARG;
    if (!q1 || !k1 || !q2 || !k2 || !kl || !lse1 || !lse2 || !dkl || !dq || !dk || !workspace)
        return STREAMKL_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, NQ, NK, d, scale, causal);
    if (rc) return rc;
    if (workspace_bytes < streamkl_bwd_workspace_bytes(B, Hq, Hkv, NQ, NK, d)) return STREAMKL_ERR_INVALID_ARG;
    const void* ptrs[] = {q1, k1, q2, k2, kl, lse1, lse2, dkl, dq, dk, workspace};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return STREAMKL_ERR_UNSUPPORTED;
    const bool shared = (k1 == k2);
    CUtensorMap mq1, mq2, mk1, mk2;
    if ((rc = make_map(&mq1, q1, (long long)B * Hq, NQ, d))) return rc;
    if ((rc = make_map(&mq2, q2, (long long)B * Hq, NQ, d))) return rc;
    if ((rc = make_map(&mk1, k1, (long long)B * Hkv, NK, d))) return rc;
    if ((rc = make_map(&mk2, k2, (long long)B * Hkv, NK, d))) return rc;
    skl::BwdParams p;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.NQ = NQ; p.NK = NK;
    p.causal = causal ? 1 : 0;
    p.nkt = (NK + 127) / 128;
    p.nqt = (NQ + 127) / 128;
    p.sl2 = scale * 1.4426950408889634f;
    p.scale = scale;
    p.kl = kl; p.lse1 = lse1; p.lse2 = lse2; p.dkl = dkl;
    p.dk_ws = static_cast<float*>(workspace);
    p.dq = dq;
    p.splits = bwd_splits(B, Hq, Hkv, NQ, NK, d);
    const int hp = bwd_heads_per_cta(Hq, Hkv, d);
    {
        int used;
        split_ranges(NK, p.splits, &p.kps, &used);
        p.splits = used;
    }
    p.dq_ws = p.splits > 1 ? p.dk_ws + bwd_dk_bytes(B, Hkv, NK, d) / sizeof(float) : nullptr;
    const long long grid = (long long)B * (Hq / hp) * p.nqt * p.splits;
    if (grid >= (1ll << 31)) return STREAMKL_ERR_UNSUPPORTED;
    const size_t ws = streamkl_bwd_workspace_bytes(B, Hq, Hkv, NQ, NK, d);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 128) {
        return shared ? launch_bwd<128, true, 1>(mode, mq1, mq2, mk1, mk2, p, (int)grid, ws, dk, st)
                      : launch_bwd<128, false, 1>(mode, mq1, mq2, mk1, mk2, p, (int)grid, ws, dk, st);
    }
    if (hp == 2)
        return shared ? launch_bwd<64, true, 2>(mode, mq1, mq2, mk1, mk2, p, (int)grid, ws, dk, st)
                      : launch_bwd<64, false, 2>(mode, mq1, mq2, mk1, mk2, p, (int)grid, ws, dk, st);
    return shared ? launch_bwd<64, true, 1>(mode, mq1, mq2, mk1, mk2, p, (int)grid, ws, dk, st)
                  : launch_bwd<64, false, 1>(mode, mq1, mq2, mk1, mk2, p, (int)grid, ws, dk, st);
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation backward
// The scratch buffer behind streamkl_bwd_noalloc: a fixed-size static device array, so the
// entry point never allocates.  It holds whatever streamkl_bwd would keep in its workspace:
// the fp32 dK accumulator, plus the fp32 dQ partial sums when the key-range split is chosen.
// Host code must not pass `g_noalloc_scratch` itself to a kernel (on the host that name is
// only a stand-in for the symbol); it passes the device address that cudaGetSymbolAddress
// returns, looked up with the device current.
static __device__ __align__(256) float g_noalloc_scratch[STREAMKL_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {

std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (ids are never reused, unlike
// context handles), or 0 when there is none yet or the driver cannot say.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool looked = false;
    if (!looked) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        looked = true;
    }
    if (!get_cur || !get_id) return 0;
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_cur(&c) != CUDA_SUCCESS || c == nullptr || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array on the current device.  The lookup is done the first
// time a device is used, with that device current, and again whenever that device's context
// has changed since (a cudaDeviceReset destroys the context and the module with it, so the
// old address is no longer valid).  Returns nullptr and sets the error text on failure.
float* noalloc_scratch() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cuda_fail(e, "cudaGetDevice");
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        snprintf(t_last_cuda_error, sizeof(t_last_cuda_error), "device %d beyond the %d supported",
                 dev, kMaxDevices);
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    const unsigned long long ctx = current_context_id();
    if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "cudaGetSymbolAddress(scratch)");
            return nullptr;
        }
        g_noalloc_ptr[dev] = static_cast<float*>(p);
        g_noalloc_ctx[dev] = current_context_id();   // the lookup made the context current
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int streamkl_bwd_noalloc(int mode, const uint16_t* q1, const uint16_t* k1,
                                    const uint16_t* q2, const uint16_t* k2, const float* kl,
                                    const float* lse1, const float* lse2, const float* dkl, int B,
                                    int Hq, int Hkv, int NQ, int NK, int d, float scale, int causal,
                                    uint16_t* dq, uint16_t* dk, void* stream) {
    if (mode != 1 && mode != 2) return STREAMKL_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, NQ, NK, d, scale, causal);
    if (rc) return rc;
    const size_t need = streamkl_bwd_workspace_bytes(B, Hq, Hkv, NQ, NK, d);
    if (need == 0 || need > STREAMKL_NOALLOC_SCRATCH_BYTES) {
        snprintf(t_last_cuda_error, sizeof(t_last_cuda_error),
                 "streamkl_bwd_noalloc: needs %zu bytes of scratch, the built-in buffer holds %zu",
                 need, (size_t)STREAMKL_NOALLOC_SCRATCH_BYTES);
        return STREAMKL_ERR_UNSUPPORTED;
    }
    float* ws = noalloc_scratch();
    if (!ws) return STREAMKL_ERR_CUDA;
    return streamkl_bwd(mode, q1, k1, q2, k2, kl, lse1, lse2, dkl, B, Hq, Hkv, NQ, NK, d, scale,
                        causal, dq, dk, ws, need, stream);
}
