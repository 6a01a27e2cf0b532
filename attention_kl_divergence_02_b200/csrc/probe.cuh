// probe.cuh -- throughput probe of the two exponential paths the kernels use: the
// exponential unit (ex2.approx on the MUFU) and the FMA-pipe polynomial ex2_poly2.  The
// StreamKL forward spends two exponentials per (row, key) pair and has no second GEMM to
// amortise them (StreamKL technical summary, gist.science, Portuguese, "1. Formulação
// Online"), so the rate of these two paths, not the tensor core, sets its floor; the bench
// divides a kernel's exponential count by the rates measured here.
//
// Every thread runs kChains independent recurrences y <- 2^(c - y/2) (values stay in
// (0.5, 2], so neither path over- or underflows); each step is one exponential and one FMA
// that forms its argument.  Nothing else is in the loop, and the sum of the chains goes to a
// store that the host never enables, so the compiler must keep every exponential.
#pragma once

#include "sm100.cuh"

namespace skl {

constexpr int kProbeChains = 8;
constexpr int kProbeThreads = 256;

template <int KIND>   // 0: MUFU ex2.approx; 1: ex2_poly2 on the FMA/ALU pipes
__global__ void __launch_bounds__(kProbeThreads)
streamkl_probe_exp2_kernel(int iters, int write, float* sink) {
    float y[kProbeChains];
#pragma unroll
    for (int k = 0; k < kProbeChains; ++k) y[k] = 1.0f + 0.01f * (float)((threadIdx.x + k) & 7);
#pragma unroll 1
    for (int i = 0; i < iters; ++i) {
        if (KIND == 0) {
#pragma unroll
            for (int k = 0; k < kProbeChains; ++k) y[k] = ex2(fmaf(y[k], -0.5f, 0.125f));
        } else {
#pragma unroll
            for (int k = 0; k < kProbeChains; k += 2) {
                const float2 u = __ffma2_rn(make_float2(y[k], y[k + 1]), make_float2(-0.5f, -0.5f),
                                            make_float2(0.125f, 0.125f));
                const float2 e = ex2_poly2(u);
                y[k] = e.x;
                y[k + 1] = e.y;
            }
        }
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kProbeChains; ++k) s += y[k];
    if (write) sink[blockIdx.x * kProbeThreads + threadIdx.x] = s;
}

// y[i] = 2^x[i] by one of the kernels' two exponential paths (KIND 0: ex2.approx on the
// exponential unit; 1: the FMA-pipe polynomial ex2_poly2), for checking their accuracy.
template <int KIND>
__global__ void __launch_bounds__(256)
streamkl_eval_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
    for (long long i = 2 * (blockIdx.x * (long long)blockDim.x + threadIdx.x); i < n;
         i += 2 * (long long)gridDim.x * blockDim.x) {
        const float2 u = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
        const float2 e = KIND == 0 ? make_float2(ex2(u.x), ex2(u.y)) : ex2_poly2(u);
        y[i] = e.x;
        if (i + 1 < n) y[i + 1] = e.y;
    }
}

// Effective SM clock.  Under the board's power cap the SM clock drops below its maximum for
// as long as heavy kernels run, and a sampled clock reading can miss it; clock64 counts the
// cycles an SM actually runs.  One thread records (globaltimer ns, clock64) pairs every
// interval_ns for duration_ns, sleeping in between, so that it can share an SM with the
// kernels being timed (one warp, no shared memory, few registers).  out[0] = pairs written,
// pair i at out[2 + 2i], out[3 + 2i].  Bounded by the duration and by an iteration cap.
constexpr long long kClockMaxIters = 1LL << 27;

__global__ void __launch_bounds__(32)
streamkl_probe_clock_kernel(long long duration_ns, long long interval_ns, int max_pairs,
                            long long* out) {
    if (threadIdx.x != 0) return;
    const long long t0 = (long long)globaltimer();
    long long next = t0;
    int n = 0;
    for (long long it = 0; it < kClockMaxIters && n < max_pairs; ++it) {
        const long long t = (long long)globaltimer();
        if (t - t0 > duration_ns) break;
        if (t >= next) {
            out[2 + 2 * n] = t;
            out[3 + 2 * n] = clock64();
            ++n;
            next = t + interval_ns;
        } else {
            __nanosleep(500);
        }
    }
    out[0] = n;
    out[1] = 0;
}

}  // namespace skl
