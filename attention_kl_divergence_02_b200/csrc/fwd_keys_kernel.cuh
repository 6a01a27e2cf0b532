// fwd_keys_kernel.cuh -- StreamKL forward for a few query rows (decoding), keys as MMA rows.
//
// Same result as fwd_kernel.cuh: per query row KL(P1 || P2) through the five running scalars
// m1, l1, m2, l2, acc (StreamKL technical summary, gist.science, Portuguese, "1. Formulação
// Online (Passagem Forward)"), with the key ranges of the split-K variant ("3. Otimizações de
// Kernel de GPU": for small N_Q the keys, not the queries, carry the parallelism).  With at
// most 8 query rows a 128-row MMA over query rows would spend 127 of its rows on nothing, so
// here the keys are the MMA's rows: per 128-key tile
//     S^T = K [Q1 | Q2]^T      (M = 128 keys, N = 32: Q1 rows then Q2 rows, each padded to
//                              16 with zero rows, K = d)
// one MMA instruction per 16 columns of d; the tensor work per key is 1/8 of a 128-row tile's
// and the kernel streams the keys at memory speed.  Thread k of the statistics warpgroup owns
// key lane k of every tile: it keeps, per query row, its own online state over the keys it
// sees (one key per tile), and the 128 lanes' states are combined once at the end with the
// same rescaling the recurrence applies (max of the maxima, sums scaled by 2^(m - M)).
//
// Roles (256 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2-3
// idle, warps 4-7 statistics (thread = key lane).  About 105 KiB of shared memory at d = 128,
// so two CTAs share an SM.
#pragma once

#include "sm100.cuh"
#include "fwd_kernel.cuh"

namespace skl {

constexpr int kKeysThreads = 256;

template <int D>
struct KeysCfg {
    static constexpr int kBoxes = D / 64;
    static constexpr int kKBox = 128 * 128;                 // 128 keys x 64 bf16
    static constexpr int kTile = kBoxes * kKBox;            // one 128-key tile
    static constexpr int kQBox = 32 * 128;                  // 16 Q1 rows + 16 Q2 rows x 64 bf16
    static constexpr int kSlots = (D == 128) ? 3 : 6;
    static constexpr int kQ = 0;                            // Q box b at kQ + b*kQBox
    static constexpr int kK = 8192;                         // key slot s at kK + s*kTile
    static constexpr int kMerge = kK + kSlots * kTile;      // 4 warps x 8 rows x 6 floats
    static constexpr int kBar = kMerge + 4 * 8 * 6 * 4;
    static constexpr int Q_FULL = 0;
    static constexpr int K_FULL = 1;                        // + s
    static constexpr int K_EMPTY = 1 + kSlots;              // + s
    static constexpr int S_FULL = 1 + 2 * kSlots;           // + buffer
    static constexpr int S_FREE = S_FULL + 2;               // + buffer
    static constexpr int DONE = S_FULL + 4;
    static constexpr int MERGE = S_FULL + 5;
    static constexpr int kNumBars = MERGE + 1;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kSmem = kMisc + 16 + 1024;
};

// One online step of a lane's state for one query row and one key (base-2 scores s1, s2 =
// raw * scale * log2 e; diff = raw s1 - raw s2).  SYM: also acc2, the same sum weighted by
// P2 and rescaled with m2 (the reverse direction's term, negated).
template <bool SYM>
__device__ __forceinline__ void keys_update(float s1, float s2, float diff, float& m1, float& l1,
                                            float& m2, float& l2, float& acc, float& acc2) {
    const float n1 = fmaxf(m1, s1);
    const float n2 = fmaxf(m2, s2);
    const float a1 = ex2(m1 - n1), e1 = ex2(s1 - n1);
    const float a2 = ex2(m2 - n2), e2 = ex2(s2 - n2);
    l1 = fmaf(l1, a1, e1);
    acc = fmaf(acc, a1, e1 * diff);
    l2 = fmaf(l2, a2, e2);
    if (SYM) acc2 = fmaf(acc2, a2, e2 * diff);
    m1 = n1;
    m2 = n2;
}

// Combines state b into state a (both over disjoint key sets).
template <bool SYM>
__device__ __forceinline__ void keys_combine(float& m1, float& l1, float& m2, float& l2, float& acc,
                                             float& acc2, float bm1, float bl1, float bm2, float bl2,
                                             float bacc, float bacc2) {
    const float M1 = fmaxf(m1, bm1), M2 = fmaxf(m2, bm2);
    const float ea = ex2(m1 - M1), eb = ex2(bm1 - M1);
    const float fa = ex2(m2 - M2), fb = ex2(bm2 - M2);
    l1 = fmaf(l1, ea, bl1 * eb);
    acc = fmaf(acc, ea, bacc * eb);
    l2 = fmaf(l2, fa, bl2 * fb);
    if (SYM) acc2 = fmaf(acc2, fa, bacc2 * fb);
    m1 = M1;
    m2 = M2;
}

template <int D, bool SHARED_K, int ROWS, bool SYM>
__global__ void __launch_bounds__(kKeysThreads, 2)
streamkl_fwd_keys_kernel(const __grid_constant__ CUtensorMap tmQ1, const __grid_constant__ CUtensorMap tmQ2,
                         const __grid_constant__ CUtensorMap tmK1, const __grid_constant__ CUtensorMap tmK2,
                         const FwdParams p) {
    using C = KeysCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(smem);
    const uint32_t bar0 = sb + C::kBar;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
#define BAR(i) (bar0 + 8u * (uint32_t)(i))

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int sp = blockIdx.x % p.splits;
    const int bh = blockIdx.x / p.splits;
    const int b = bh / p.Hq;
    const int h = bh % p.Hq;
    const int bhk = b * p.Hkv + h / (p.Hq / p.Hkv);
    const int nkt = (p.NK + 127) >> 7;
    const int j0 = sp * p.kps;
    const int j1 = min(nkt, j0 + p.kps);
    const int nj = max(0, j1 - j0);
    constexpr int kPerTile = SHARED_K ? 1 : 2;

    if (threadIdx.x == 0) {
        mbar_init(BAR(C::Q_FULL), 1);
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(BAR(C::K_FULL + s), 1);
            mbar_init(BAR(C::K_EMPTY + s), 1);
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(BAR(C::S_FULL + u), 1);
            mbar_init(BAR(C::S_FREE + u), 128);
        }
        mbar_init(BAR(C::DONE), 1);
        mbar_init(BAR(C::MERGE), 4);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ1);
            tma_prefetch_desc(&tmQ2);
            tma_prefetch_desc(&tmK1);
            if (!SHARED_K) tma_prefetch_desc(&tmK2);
            // query rows 0..15 of this head (rows past NQ arrive as zeros)
            mbar_arrive_expect_tx(BAR(C::Q_FULL), C::kBoxes * C::kQBox);
            for (int bx = 0; bx < C::kBoxes; ++bx) {
                tma_load_3d(sb + C::kQ + bx * C::kQBox, &tmQ1, BAR(C::Q_FULL), bx * 64, 0, bh);
                tma_load_3d(sb + C::kQ + bx * C::kQBox + 2048, &tmQ2, BAR(C::Q_FULL), bx * 64, 0, bh);
            }
            uint32_t it = 0;
            bool ok = true;
            for (int j = j0; j < j1 && ok; ++j) {
#pragma unroll
                for (int w = 0; w < kPerTile; ++w) {
                    const uint32_t s = it % C::kSlots;
                    const uint32_t n = it / C::kSlots;
                    if (n > 0 && !mbar_wait(BAR(C::K_EMPTY + s), (n - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(BAR(C::K_FULL + s), C::kTile);
                    const CUtensorMap* map = (w == 0) ? &tmK1 : &tmK2;
                    for (int bx = 0; bx < C::kBoxes; ++bx)
                        tma_load_3d(sb + C::kK + s * C::kTile + bx * C::kKBox, map, BAR(C::K_FULL + s),
                                    bx * 64, j * 128, bhk);
                    ++it;
                }
            }
            drain_wait(BAR(C::Q_FULL), 0);
            for (uint32_t s = 0; s < (uint32_t)C::kSlots; ++s) {
                if (it > s) {
                    const uint32_t fills = (it - s - 1) / C::kSlots + 1;
                    drain_wait(BAR(C::K_FULL + s), (fills - 1) & 1);
                }
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, 32, 0, 0);
            bool ok = mbar_wait(BAR(C::Q_FULL), 0, abort_flag);
            tc_fence_after();
            uint32_t it = 0;
            for (int u = 0; u < nj && ok; ++u) {
                const int buf = u & 1;
                if (u >= 2) {
                    if (!mbar_wait(BAR(C::S_FREE + buf), ((u >> 1) - 1) & 1, abort_flag)) break;
                    tc_fence_after();
                }
                const uint32_t s1 = it % C::kSlots;
                if (!mbar_wait(BAR(C::K_FULL + s1), (it / C::kSlots) & 1, abort_flag)) break;
                ++it;
                uint32_t s2 = s1;
                if (!SHARED_K) {
                    s2 = it % C::kSlots;
                    if (!mbar_wait(BAR(C::K_FULL + s2), (it / C::kSlots) & 1, abort_flag)) break;
                    ++it;
                }
                tc_fence_after();
                // S^T into TMEM columns [64*buf, +32) (and, with distinct keys, K2's product
                // into [64*buf + 32, +32)); Q1 rows are columns 0-15, Q2 rows 16-31
                const uint32_t d0 = tmem + 64 * buf;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t ka = (k >> 2) * C::kKBox + (k & 3) * 32;
                    const uint32_t qb = (k >> 2) * C::kQBox + (k & 3) * 32;
                    mma_bf16_ss(d0, sw128_desc(sb + C::kK + s1 * C::kTile + ka, 16, 1024),
                                sw128_desc(sb + C::kQ + qb, 16, 1024), idesc, k > 0);
                }
                if (!SHARED_K) {
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t ka = (k >> 2) * C::kKBox + (k & 3) * 32;
                        const uint32_t qb = (k >> 2) * C::kQBox + (k & 3) * 32;
                        mma_bf16_ss(d0 + 32, sw128_desc(sb + C::kK + s2 * C::kTile + ka, 16, 1024),
                                    sw128_desc(sb + C::kQ + qb, 16, 1024), idesc, k > 0);
                    }
                }
                mma_commit(BAR(C::S_FULL + buf));
                mma_commit(BAR(C::K_EMPTY + s1));
                if (!SHARED_K) mma_commit(BAR(C::K_EMPTY + s2));
            }
            mma_commit(BAR(C::DONE));
            drain_wait(BAR(C::DONE), 0);
        }
    } else if (warp >= 4) {
        // ================================================================ statistics
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;                  // key lane
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sl2 = p.sl2;
        float m1[ROWS], l1[ROWS], m2[ROWS], l2[ROWS], acc[ROWS], acc2[ROWS];
#pragma unroll
        for (int t = 0; t < ROWS; ++t) {
            m1[t] = -1e30f; l1[t] = 0.f; m2[t] = -1e30f; l2[t] = 0.f; acc[t] = 0.f; acc2[t] = 0.f;
        }
        bool ok = true;
        for (int u = 0; u < nj; ++u) {
            const int buf = u & 1;
            if (!mbar_wait(BAR(C::S_FULL + buf), (u >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t xa[8], ya[8];
            tmem_ld8(lane_base + 64 * buf, xa);
            tmem_ld8(lane_base + 64 * buf + (SHARED_K ? 16 : 48), ya);
            tmem_wait_ld_regs(xa, ya);
            tc_fence_before();
            mbar_arrive(BAR(C::S_FREE + buf));
            const int key = (j0 + u) * 128 + r;
            if (key < p.NK) {
#pragma unroll
                for (int t = 0; t < ROWS; ++t) {
                    if (t < p.NQ && (!p.causal || key <= t)) {
                        const float x = __uint_as_float(xa[t]), y = __uint_as_float(ya[t]);
                        keys_update<SYM>(x * sl2, y * sl2, x - y, m1[t], l1[t], m2[t], l2[t], acc[t], acc2[t]);
                    }
                }
            }
        }
        // combine the 128 lanes: within each warp by butterfly, then the four warps in smem
#pragma unroll
        for (int t = 0; t < ROWS; ++t) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float bm1 = __shfl_xor_sync(0xffffffffu, m1[t], o);
                const float bl1 = __shfl_xor_sync(0xffffffffu, l1[t], o);
                const float bm2 = __shfl_xor_sync(0xffffffffu, m2[t], o);
                const float bl2 = __shfl_xor_sync(0xffffffffu, l2[t], o);
                const float bac = __shfl_xor_sync(0xffffffffu, acc[t], o);
                const float bac2 = SYM ? __shfl_xor_sync(0xffffffffu, acc2[t], o) : 0.f;
                keys_combine<SYM>(m1[t], l1[t], m2[t], l2[t], acc[t], acc2[t], bm1, bl1, bm2, bl2, bac, bac2);
            }
        }
        float* mb = reinterpret_cast<float*>(smem + C::kMerge);   // [warp][row][6]
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < ROWS; ++t) {
                float* e = mb + (quarter * 8 + t) * 6;
                e[0] = m1[t]; e[1] = l1[t]; e[2] = m2[t]; e[3] = l2[t]; e[4] = acc[t]; e[5] = acc2[t];
            }
            mbar_arrive(BAR(C::MERGE));
        }
        if (quarter == 0) {
            ok = mbar_wait(BAR(C::MERGE), 0, abort_flag) && ok;
            const int t = lane;
            if (ok && t < ROWS && t < p.NQ) {
                float M1 = -1e30f, L1 = 0.f, M2 = -1e30f, L2 = 0.f, A = 0.f, A2 = 0.f;
                for (int w = 0; w < 4; ++w) {
                    const float* e = mb + (w * 8 + t) * 6;
                    keys_combine<SYM>(M1, L1, M2, L2, A, A2, e[0], e[1], e[2], e[3], e[4], e[5]);
                }
                const size_t o = (size_t)bh * p.NQ + t;
                if (p.splits > 1) {
                    const size_t R = (size_t)p.B * p.Hq * p.NQ;
                    float* dst = p.part + (size_t)sp * 5 * R + o;
                    dst[0] = M1;
                    dst[R] = L1;
                    dst[2 * R] = M2;
                    dst[3 * R] = L2;
                    dst[4 * R] = A;
                } else {
                    const float LN2 = 0.6931471805599453f;
                    const float lg1 = log2f(L1), lg2 = log2f(L2);
                    p.lse1[o] = (M1 + lg1) * LN2;
                    p.lse2[o] = (M2 + lg2) * LN2;
                    p.kl[o] = p.scale * A / L1 + ((M2 - M1) + (lg2 - lg1)) * LN2;
                    if (SYM) p.kl21[o] = -p.scale * A2 / L2 + ((M1 - M2) + (lg1 - lg2)) * LN2;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
#undef BAR
}

}  // namespace skl
