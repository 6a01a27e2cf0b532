// fwd_kernel.cuh -- StreamKL forward on sm_100a.
//
// One CTA owns 256 query rows of one (batch, query head): two 128-row tiles t = 0, 1.
// Key tiles of 128 keys stream through a ring of shared-memory slots filled by TMA.  For
// every key tile the tensor core computes S1 = Q1 K1^T and S2 = Q2 K2^T for both query
// tiles into TMEM (fp32, lane = query row, column = key), and two 128-thread statistics
// warpgroups (one thread per row) fold it into the rows' five running scalars
//   m1, l1, m2, l2, acc
// (StreamKL technical summary, gist.science, Portuguese, "1. Formulação Online (Passagem
// Forward)"), rescaling l1, acc and l2 by 2^(m_old - m_new) whenever a maximum grows (the
// online correction of the FlashAttention lecture notes, hackmd, "4. Flash Attention 的核心
// 數學重構").  At the end it writes KL = acc/l1 + LSE2 - LSE1 and both LSEs.  Causal key
// tiles past the diagonal are never loaded or multiplied.
//
// Roles (384 threads):  warp 0 = TMA producer, warp 1 = TMEM allocator + MMA issuer,
// warps 2-3 idle, warps 4-7 and 8-11 = statistics warpgroups g = 0, 1.  With two query tiles
// warpgroup g folds key columns [64g, 64g + 64) of both tiles (one state per row and tile);
// with one query tile the two warpgroups take alternate key tiles of it, each in its own
// TMEM half; with at most 32 query rows the rows sit in all four lane quarters and each warp
// folds one 32-column chunk.  The partial states of a row are combined in the CTA at the
// end.  Warp w may touch TMEM lanes 32*(w%4) .. 32*(w%4)+31, so each statistics warp owns
// the 32 rows that live in its lane quarter.
//
// Scores are kept in base-2 units: u = s_raw * scale * log2(e), where s_raw = <q, k>.
//
// Split-K (for few query rows and many keys, where one CTA per query block leaves most SMs
// idle; the technical summary's "3. Otimizações de Kernel de GPU" names it for small N_Q):
// with splits > 1 the key tiles are cut into ranges of kps tiles, CTA (block, split) folds
// only its range, and instead of finishing it stores the five scalars of each row; the
// merge kernel below combines the ranges exactly (each rescaled to the common maximum, the
// same correction the online recurrence applies tile by tile).  The merge is launched as a
// programmatic dependent of this kernel and waits for it with griddepcontrol.wait.
//
// At most 8 query rows run in fwd_keys_kernel.cuh instead (keys as the MMA's rows); the
// symmetric variant (SYM) adds the reverse direction's running sum to either kernel.
#pragma once

#include "sm100.cuh"

namespace skl {

struct FwdParams {
    int B, Hq, Hkv, NQ, NK;
    int causal;
    int n_qblk;    // ceil(NQ / 256)
    float sl2;     // scale * log2(e)
    float scale;
    float* kl;
    float* lse1;
    float* lse2;
    int rep4;      // NQ <= 32: the query tile holds rows 0..31 in each 32-lane quarter
    int splits;    // key ranges per query block (1 = no split)
    int kps;       // key tiles per range
    float* part;   // splits > 1: partial state [splits][5][B*Hq*NQ]: m1, l1, m2, l2, acc
    float* kl21;   // symmetric variant only: KL(P2 || P1) per row (else unused)
};

constexpr int kFwdThreads = 384;

template <int D>
struct FwdCfg {
    static constexpr int kTile = 128 * D * 2;       // bytes of one 128-row bf16 tile
    static constexpr int kBoxes = D / 64;           // 64-column (128-byte) TMA boxes per tile
    static constexpr int kBox = 128 * 128;          // bytes of one box: 128 rows x 128 bytes
    static constexpr int kSlots = (D == 128) ? 3 : 6;
    static constexpr int kQ1 = 0;                   // Q1 tile t at kQ1 + t*kTile
    static constexpr int kQ2 = 2 * kTile;           // Q2 tile t at kQ2 + t*kTile
    static constexpr int kK = 4 * kTile;            // key slot s at kK + s*kTile
    static constexpr int kBar = kK + kSlots * kTile;
    // barrier indices
    static constexpr int Q_FULL = 0;                // + t
    static constexpr int K_FULL = 2;                // + s
    static constexpr int K_EMPTY = 2 + kSlots;      // + s
    static constexpr int S_FULL = 2 + 2 * kSlots;   // + t
    static constexpr int S_FREE = S_FULL + 2;       // + t
    static constexpr int DONE = S_FREE + 2;
    static constexpr int MERGE = DONE + 1;          // partial states of a row are stored
    static constexpr int kNumBars = MERGE + 1;
    static constexpr int kMisc = kBar + kNumBars * 8;   // tmem address, abort flag
    static constexpr int kSmem = kMisc + 16 + 1024;     // + slack for 1024-byte alignment
};


// Column pairs (bit p = columns 2p, 2p+1 of a 32-column chunk) whose exponentials go to
// the FMA-pipe polynomial instead of the exponential unit, for S1 and for S2, so that the
// two pipes share the exponentials of a chunk.
// Default: a quarter of each (pairs 1, 5, 9, 13 of S1 and 3, 7, 11, 15 of S2, spread so
// the polynomial work interleaves with the exponential unit's); chosen by timing the
// headline forward (2.75 ms with none, 2.61 ms with this split, slower with more; at d = 64
// a third or a half on the FMA pipe is slower too: 5.05 -> 5.23 / 5.47 ms on B4 Hq32 NK32768).
#ifndef SKL_FWD_EMU1
#define SKL_FWD_EMU1 0x2222u
#endif
#ifndef SKL_FWD_EMU2
#define SKL_FWD_EMU2 0x8888u
#endif
constexpr uint32_t kEmu1 = SKL_FWD_EMU1;
constexpr uint32_t kEmu2 = SKL_FWD_EMU2;

// Fold 32 columns of one row, all valid keys, into the running scalars (x = S1 raw
// scores, y = S2 raw).  Adjacent columns are processed as fp32x2 pairs: they are adjacent
// registers of one TMEM load, so each add/FMA instruction serves two columns.
//
// SYM: also accumulate acc2 = sum 2^(u2 - m2) (s1 - s2), rescaled with m2, whose negation over
// l2 is the reverse direction's (s2 - s1) term, so that one pass gives both KL(P1 || P2) and
// KL(P2 || P1) (their sum is the symmetric divergence).
template <bool SYM>
__device__ __forceinline__ void fold_chunk_full(const uint32_t (&xa)[32], const uint32_t (&ya)[32],
                                                float sl2, float& m1, float& l1, float& m2,
                                                float& l2, float& acc, float& acc2) {
    float mx1 = __uint_as_float(xa[0]), mx2 = __uint_as_float(ya[0]);
#pragma unroll
    for (int k = 1; k < 31; k += 2) {
        mx1 = fmax3(mx1, __uint_as_float(xa[k]), __uint_as_float(xa[k + 1]));
        mx2 = fmax3(mx2, __uint_as_float(ya[k]), __uint_as_float(ya[k + 1]));
    }
    mx1 = fmaxf(mx1, __uint_as_float(xa[31]));
    mx2 = fmaxf(mx2, __uint_as_float(ya[31]));
    const float m1n = fmaxf(m1, mx1 * sl2);
    const float m2n = fmaxf(m2, mx2 * sl2);
    const float a1 = ex2(m1 - m1n);
    const float a2 = ex2(m2 - m2n);
    m1 = m1n;
    m2 = m2n;
    const float2 sl = make_float2(sl2, sl2);
    const float2 nm1 = make_float2(-m1n, -m1n);
    const float2 nm2 = make_float2(-m2n, -m2n);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    float2 L1[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 L2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 AC[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 AC2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int pr = 0; pr < 16; ++pr) {
        const float2 xk = make_float2(__uint_as_float(xa[2 * pr]), __uint_as_float(xa[2 * pr + 1]));
        const float2 yk = make_float2(__uint_as_float(ya[2 * pr]), __uint_as_float(ya[2 * pr + 1]));
        const float2 u1 = __ffma2_rn(xk, sl, nm1);
        const float2 u2 = __ffma2_rn(yk, sl, nm2);
        const float2 e1 = ((kEmu1 >> pr) & 1u) ? ex2_poly2(u1) : make_float2(ex2(u1.x), ex2(u1.y));
        const float2 e2 = ((kEmu2 >> pr) & 1u) ? ex2_poly2(u2) : make_float2(ex2(u2.x), ex2(u2.y));
        L1[pr & 1] = __fadd2_rn(L1[pr & 1], e1);
        L2[pr & 1] = __fadd2_rn(L2[pr & 1], e2);
        const float2 dk = __ffma2_rn(yk, neg1, xk);
        AC[pr & 1] = __ffma2_rn(e1, dk, AC[pr & 1]);
        if (SYM) AC2[pr & 1] = __ffma2_rn(e2, dk, AC2[pr & 1]);
    }
    const float2 L1s = __fadd2_rn(L1[0], L1[1]);
    const float2 L2s = __fadd2_rn(L2[0], L2[1]);
    const float2 ACs = __fadd2_rn(AC[0], AC[1]);
    l1 = fmaf(l1, a1, L1s.x + L1s.y);
    acc = fmaf(acc, a1, ACs.x + ACs.y);
    l2 = fmaf(l2, a2, L2s.x + L2s.y);
    if (SYM) {
        const float2 AC2s = __fadd2_rn(AC2[0], AC2[1]);
        acc2 = fmaf(acc2, a2, AC2s.x + AC2s.y);
    }
}

// Same fold for a chunk with invalid columns (bit k of `valid` clear): those are left out of
// the maxima and of every sum, including the (s1 - s2) term, which would be NaN there.
template <bool SYM>
__device__ __forceinline__ void fold_chunk_masked(const uint32_t (&xa)[32], const uint32_t (&ya)[32],
                                                  uint32_t valid, float sl2, float& m1, float& l1,
                                                  float& m2, float& l2, float& acc, float& acc2) {
    float x[32], y[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const bool ok = (valid >> k) & 1u;
        x[k] = ok ? __uint_as_float(xa[k]) : -INFINITY;
        y[k] = ok ? __uint_as_float(ya[k]) : -INFINITY;
    }
    float mx1 = x[0], mx2 = y[0];
#pragma unroll
    for (int k = 1; k < 32; ++k) {
        mx1 = fmaxf(mx1, x[k]);
        mx2 = fmaxf(mx2, y[k]);
    }
    const float m1n = fmaxf(m1, mx1 * sl2);
    const float m2n = fmaxf(m2, mx2 * sl2);
    const float a1 = ex2(m1 - m1n);
    const float a2 = ex2(m2 - m2n);
    m1 = m1n;
    m2 = m2n;
    float sl1 = 0.f, sl2v = 0.f, sac = 0.f, sac2 = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float e1 = ex2(fmaf(x[k], sl2, -m1n));
        const float e2 = ex2(fmaf(y[k], sl2, -m2n));
        const float diff = ((valid >> k) & 1u) ? x[k] - y[k] : 0.f;
        sl1 += e1;
        sl2v += e2;
        sac = fmaf(e1, diff, sac);
        if (SYM) sac2 = fmaf(e2, diff, sac2);
    }
    l1 = fmaf(l1, a1, sl1);
    acc = fmaf(acc, a1, sac);
    l2 = fmaf(l2, a2, sl2v);
    if (SYM) acc2 = fmaf(acc2, a2, sac2);
}

template <int D, bool SHARED_K, bool SYM>
__global__ void __launch_bounds__(kFwdThreads, 1)
streamkl_fwd_kernel(const __grid_constant__ CUtensorMap tmQ1, const __grid_constant__ CUtensorMap tmQ2,
                    const __grid_constant__ CUtensorMap tmK1, const __grid_constant__ CUtensorMap tmK2,
                    const FwdParams p) {
    using C = FwdCfg<D>;
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

    // ---- work unit: heaviest causal query blocks are handed out first; the key ranges of a
    // query block are neighbours in the grid
    const int BH = p.B * p.Hq;
    const int sp = blockIdx.x % p.splits;
    const int ub = blockIdx.x / p.splits;
    const int unit = ub / BH;
    const int bh = ub % BH;
    const int qb = p.causal ? (p.n_qblk - 1 - unit) : unit;
    const int b = bh / p.Hq;
    const int h = bh % p.Hq;
    const int bhk = b * p.Hkv + h / (p.Hq / p.Hkv);
    const int nkt_all = (p.NK + 127) >> 7;
    int q0[2], nkt[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        q0[t] = qb * 256 + t * 128;
        if (q0[t] >= p.NQ) {
            nkt[t] = 0;
        } else if (p.causal) {
            const int last_row = min(q0[t] + 127, p.NQ - 1);
            nkt[t] = min(nkt_all, (last_row >> 7) + 1);
        } else {
            nkt[t] = nkt_all;
        }
    }
    const int ntiles = nkt[1] > 0 ? 2 : 1;
    // this CTA's key tiles: [j0, jend[t]) for query tile t (empty when the range starts past
    // the tile's causal end)
    const int j0 = sp * p.kps;
    int jend[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) jend[t] = max(j0, min(nkt[t], j0 + p.kps));
    const int nj = max(jend[0], jend[1]);
    // One query tile and at least two key tiles: the two TMEM halves and both statistics
    // warpgroups take alternate key tiles of tile 0, so the MMAs of one key tile run while
    // the other is folded.  Each row then has (alt ? 2 : 1) * (rep4 ? 4 : 1) partial states,
    // merged in the CTA at the end.
    const bool alt = (ntiles == 1) && (nj - j0 > 1);
    const int n_contrib = (alt ? 2 : 1) * (p.rep4 ? 4 : 1);
    // Two query tiles: warpgroup g folds key columns [64g, 64g + 64) of BOTH tiles (a thread
    // can read its row in either tile's TMEM columns).  Tile t's S is then free as soon as
    // both warpgroups have loaded their two chunks of it, and its next MMAs run while the
    // warpgroups fold the other tile.  The two column halves of a row merge at the end.
    const bool split = (ntiles == 2);

    // ---- setup
    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(BAR(C::Q_FULL + t), 1);
            mbar_init(BAR(C::S_FULL + t), 1);
            mbar_init(BAR(C::S_FREE + t), split ? 256 : 128);
        }
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(BAR(C::K_FULL + s), 1);
            mbar_init(BAR(C::K_EMPTY + s), 1);
        }
        mbar_init(BAR(C::DONE), 1);
        mbar_init(BAR(C::MERGE), (alt || split) ? 256 : 128);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
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
            for (int t = 0; t < ntiles; ++t) {
                mbar_arrive_expect_tx(BAR(C::Q_FULL + t), 2 * C::kTile);
                for (int bx = 0; bx < C::kBoxes; ++bx) {
                    // rep4: four 32-row copies (4 KiB each; the swizzle pattern repeats every
                    // 8 rows, so each copy sits exactly where rows 32c.. of a 128-row box go)
                    for (int c = 0; c < (p.rep4 ? 4 : 1); ++c) {
                        const uint32_t o = t * C::kTile + bx * C::kBox + c * 4096;
                        tma_load_3d(sb + C::kQ1 + o, &tmQ1, BAR(C::Q_FULL + t), bx * 64, q0[t], bh);
                        tma_load_3d(sb + C::kQ2 + o, &tmQ2, BAR(C::Q_FULL + t), bx * 64, q0[t], bh);
                    }
                }
            }
            uint32_t it = 0;
            bool ok = true;
            for (int j = j0; j < nj && ok; ++j) {
#pragma unroll
                for (int w = 0; w < (SHARED_K ? 1 : 2); ++w) {
                    const uint32_t s = it % C::kSlots;
                    const uint32_t n = it / C::kSlots;
                    if (n > 0 && !mbar_wait(BAR(C::K_EMPTY + s), (n - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(BAR(C::K_FULL + s), C::kTile);
                    const CUtensorMap* map = (w == 0) ? &tmK1 : &tmK2;
                    for (int bx = 0; bx < C::kBoxes; ++bx)
                        tma_load_3d(sb + C::kK + s * C::kTile + bx * C::kBox, map, BAR(C::K_FULL + s),
                                    bx * 64, j * 128, bhk);
                    ++it;
                }
            }
            // drain: every copy this thread started must land before the CTA exits
            for (int t = 0; t < ntiles; ++t) drain_wait(BAR(C::Q_FULL + t), 0);
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
            constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 0);
            bool ok = true;
            for (int t = 0; t < ntiles && ok; ++t) ok = mbar_wait(BAR(C::Q_FULL + t), 0, abort_flag);
            tc_fence_after();
            uint32_t it = 0;
            for (int j = j0; j < nj && ok; ++j) {
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
                const int u = j - j0;
                for (int t = 0; t < (alt ? 1 : ntiles); ++t) {
                    // TMEM half h (= statistics warpgroup h) and how often it was used before
                    int h, use;
                    if (alt) {
                        h = u & 1;
                        use = u >> 1;
                    } else {
                        if (j >= jend[t]) continue;
                        h = t;
                        use = u;
                    }
                    if (use > 0) {
                        if (!mbar_wait(BAR(C::S_FREE + h), (use - 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    const uint32_t d1 = tmem + h * 256;
                    const uint32_t d2 = d1 + 128;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t off = (k >> 2) * C::kBox + (k & 3) * 32;
                        mma_bf16_ss(d1, sw128_desc(sb + C::kQ1 + t * C::kTile + off, 16, 1024),
                                    sw128_desc(sb + C::kK + s1 * C::kTile + off, 16, 1024), idesc,
                                    k > 0);
                    }
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t off = (k >> 2) * C::kBox + (k & 3) * 32;
                        mma_bf16_ss(d2, sw128_desc(sb + C::kQ2 + t * C::kTile + off, 16, 1024),
                                    sw128_desc(sb + C::kK + s2 * C::kTile + off, 16, 1024), idesc,
                                    k > 0);
                    }
                    mma_commit(BAR(C::S_FULL + h));
                }
                mma_commit(BAR(C::K_EMPTY + s1));
                if (!SHARED_K) mma_commit(BAR(C::K_EMPTY + s2));
            }
            // drain: every MMA this thread issued must finish before TMEM is released
            mma_commit(BAR(C::DONE));
            drain_wait(BAR(C::DONE), 0);
        }
    } else if (warp >= 4) {
        // ================================================================ statistics
        const int g = (warp - 4) >> 2;          // warpgroup = TMEM half it reads
        const int t = alt ? 0 : g;              // query tile whose rows it folds
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const bool rep4 = p.rep4 != 0;
        // rep4: every quarter holds rows 0..31, and warp `quarter` folds only key columns
        // [32*quarter, 32*quarter + 32) of each tile; the four states are merged at the end
        const int c_lo = rep4 ? quarter : 0;
        const int c_hi = rep4 ? quarter + 1 : 4;
        // writes one finished row: its partial state (split-K) or KL, LSE1, LSE2
        constexpr int kF = SYM ? 6 : 5;   // fields of a row's state in the merge buffers
        auto write_row = [&](int i, float m1, float l1, float m2, float l2, float acc, float acc2) {
            if (p.splits > 1) {
                const size_t R = (size_t)p.B * p.Hq * p.NQ;
                float* dst = p.part + (size_t)sp * 5 * R + (size_t)bh * p.NQ + i;
                dst[0] = m1;
                dst[R] = l1;
                dst[2 * R] = m2;
                dst[3 * R] = l2;
                dst[4 * R] = acc;
            } else {
                const float LN2 = 0.6931471805599453f;
                const float lg1 = log2f(l1);
                const float lg2 = log2f(l2);
                const size_t o = (size_t)bh * p.NQ + i;
                p.lse1[o] = (m1 + lg1) * LN2;
                p.lse2[o] = (m2 + lg2) * LN2;
                p.kl[o] = p.scale * acc / l1 + ((m2 - m1) + (lg2 - lg1)) * LN2;
                if (SYM) p.kl21[o] = -p.scale * acc2 / l2 + ((m1 - m2) + (lg1 - lg2)) * LN2;
            }
        };
        if (split && g < 2) {
            const float sl2 = p.sl2;
            const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
            float st[2][6];
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2) {
                st[t2][0] = -1e30f; st[t2][1] = 0.f; st[t2][2] = -1e30f; st[t2][3] = 0.f; st[t2][4] = 0.f;
                st[t2][5] = 0.f;
            }
            bool ok = true;
            for (int j = j0; j < nj && ok; ++j) {
#pragma unroll
                for (int t2 = 0; t2 < 2; ++t2) {
                    if (!ok || j >= jend[t2]) continue;
                    if (!mbar_wait(BAR(C::S_FULL + t2), (j - j0) & 1, abort_flag)) {
                        ok = false;
                        continue;
                    }
                    tc_fence_after();
                    if (q0[t2] + quarter * 32 >= p.NQ) {   // no valid row in this warp
                        tc_fence_before();
                        mbar_arrive(BAR(C::S_FREE + t2));
                        continue;
                    }
                    const int i2 = q0[t2] + r;
                    const uint32_t tS1 = tmem + lanes + (uint32_t)(t2 * 256);
                    const uint32_t tS2 = tS1 + 128;
                    const int kb = j * 128;
                    const bool masked = (kb + 128 > p.NK) || (p.causal && kb + 127 > q0[t2]);
#pragma unroll 1
                    for (int c = 2 * g; c < 2 * g + 2; ++c) {
                        uint32_t xa[32], ya[32];
                        tmem_ld32(tS1 + c * 32, xa);
                        tmem_ld32(tS2 + c * 32, ya);
                        tmem_wait_ld();
                        if (c == 2 * g + 1) {
                            tc_fence_before();
                            mbar_arrive(BAR(C::S_FREE + t2));
                        }
                        if (!masked) {
                            fold_chunk_full<SYM>(xa, ya, sl2, st[t2][0], st[t2][1], st[t2][2], st[t2][3],
                                                 st[t2][4], st[t2][5]);
                        } else {
                            const int k0 = kb + c * 32;
                            int lim = p.NK - k0;
                            if (p.causal) lim = min(lim, i2 - k0 + 1);
                            const uint32_t valid = lim >= 32 ? 0xFFFFFFFFu
                                                 : (lim <= 0 ? 0u : ((1u << lim) - 1u));
                            fold_chunk_masked<SYM>(xa, ya, valid, sl2, st[t2][0], st[t2][1], st[t2][2],
                                                   st[t2][3], st[t2][4], st[t2][5]);
                        }
                    }
                }
            }
            // the two column halves of every row meet in key slot 0 once every MMA (hence
            // every key copy) is complete; warpgroup 0 combines them and writes both tiles
            ok = mbar_wait(BAR(C::DONE), 0, abort_flag) && ok;
            float* mb = reinterpret_cast<float*>(smem + C::kK);
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2)
#pragma unroll
                for (int f = 0; f < kF; ++f) mb[((t2 * 2 + g) * kF + f) * 128 + r] = st[t2][f];
            mbar_arrive(BAR(C::MERGE));
            if (g == 0) {
                ok = mbar_wait(BAR(C::MERGE), 0, abort_flag) && ok;
#pragma unroll
                for (int t2 = 0; t2 < 2; ++t2) {
                    const float* a0 = mb + (t2 * 2 + 0) * kF * 128 + r;
                    const float* a1 = mb + (t2 * 2 + 1) * kF * 128 + r;
                    const float M1 = fmaxf(a0[0], a1[0]);
                    const float M2 = fmaxf(a0[2 * 128], a1[2 * 128]);
                    const float e10 = ex2(a0[0] - M1), e11 = ex2(a1[0] - M1);
                    const float e20 = ex2(a0[2 * 128] - M2), e21 = ex2(a1[2 * 128] - M2);
                    const float L1 = fmaf(a0[128], e10, a1[128] * e11);
                    const float A = fmaf(a0[4 * 128], e10, a1[4 * 128] * e11);
                    const float L2 = fmaf(a0[3 * 128], e20, a1[3 * 128] * e21);
                    const float A2 = SYM ? fmaf(a0[5 * 128], e20, a1[5 * 128] * e21) : 0.f;
                    const int i2 = q0[t2] + r;
                    if (ok && i2 < p.NQ) write_row(i2, M1, L1, M2, L2, A, A2);
                }
            }
        } else if (!split && g < (alt ? 2 : ntiles)) {
            const int i = q0[t] + (rep4 ? lane : r);
            const uint32_t tS1 = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(g * 256);
            const uint32_t tS2 = tS1 + 128;
            const float sl2 = p.sl2;
            float m1 = -1e30f, l1 = 0.f, m2 = -1e30f, l2 = 0.f, acc = 0.f, acc2 = 0.f;
            bool ok = true;
            // a warp whose 32 rows all lie past NQ only keeps the barrier protocol
            const bool any_row = rep4 || q0[t] + quarter * 32 < p.NQ;
            for (int j = j0 + (alt ? g : 0); j < jend[t]; j += (alt ? 2 : 1)) {
                const int use = alt ? (j - j0) >> 1 : j - j0;
                if (!mbar_wait(BAR(C::S_FULL + g), use & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (!any_row) {
                    tc_fence_before();
                    mbar_arrive(BAR(C::S_FREE + g));
                    continue;
                }
                const int kb = j * 128;
                const bool masked = (kb + 128 > p.NK) || (p.causal && kb + 127 > q0[t]);
#pragma unroll 1
                for (int c = c_lo; c < c_hi; ++c) {
                    uint32_t xa[32], ya[32];
                    tmem_ld32(tS1 + c * 32, xa);
                    tmem_ld32(tS2 + c * 32, ya);
                    tmem_wait_ld();
                    if (c == c_hi - 1) {
                        tc_fence_before();
                        mbar_arrive(BAR(C::S_FREE + g));
                    }
                    if (!masked) {
                        fold_chunk_full<SYM>(xa, ya, sl2, m1, l1, m2, l2, acc, acc2);
                    } else {
                        const int k0 = kb + c * 32;
                        int lim = p.NK - k0;                       // keys k0 + k valid if k < lim
                        if (p.causal) lim = min(lim, i - k0 + 1);  // ... and k0 + k <= i
                        const uint32_t valid = lim >= 32 ? 0xFFFFFFFFu
                                             : (lim <= 0 ? 0u : ((1u << lim) - 1u));
                        fold_chunk_masked<SYM>(xa, ya, valid, sl2, m1, l1, m2, l2, acc, acc2);
                    }
                }
            }
            if (n_contrib > 1) {
                // The partial states of a row meet in key slot 0, reused only once every MMA
                // has completed (hence every key copy has landed and been read), and one
                // thread per row combines them like the split-K merge does.
                ok = mbar_wait(BAR(C::DONE), 0, abort_flag) && ok;
                float* mb = reinterpret_cast<float*>(smem + C::kK);
                const int rows_per = rep4 ? 32 : 128;
                const int rho = rep4 ? lane : r;
                const int kappa = (alt ? g : 0) * (rep4 ? 4 : 1) + (rep4 ? quarter : 0);
                const float st[6] = {m1, l1, m2, l2, acc, acc2};
#pragma unroll
                for (int f = 0; f < kF; ++f) mb[(kappa * kF + f) * rows_per + rho] = st[f];
                mbar_arrive(BAR(C::MERGE));
                if (g == 0 && (!rep4 || quarter == 0)) {
                    ok = mbar_wait(BAR(C::MERGE), 0, abort_flag) && ok;
                    float M1 = -1e30f, M2 = -1e30f;
                    for (int w = 0; w < n_contrib; ++w) {
                        M1 = fmaxf(M1, mb[(w * kF + 0) * rows_per + rho]);
                        M2 = fmaxf(M2, mb[(w * kF + 2) * rows_per + rho]);
                    }
                    float L1 = 0.f, L2 = 0.f, A = 0.f, A2 = 0.f;
                    for (int w = 0; w < n_contrib; ++w) {
                        const float a1 = ex2(mb[(w * kF + 0) * rows_per + rho] - M1);
                        const float a2 = ex2(mb[(w * kF + 2) * rows_per + rho] - M2);
                        L1 = fmaf(mb[(w * kF + 1) * rows_per + rho], a1, L1);
                        A = fmaf(mb[(w * kF + 4) * rows_per + rho], a1, A);
                        L2 = fmaf(mb[(w * kF + 3) * rows_per + rho], a2, L2);
                        if (SYM) A2 = fmaf(mb[(w * kF + 5) * rows_per + rho], a2, A2);
                    }
                    m1 = M1; l1 = L1; m2 = M2; l2 = L2; acc = A; acc2 = A2;
                } else {
                    ok = false;   // one thread per row writes it
                }
            }
            if (ok && i < p.NQ) write_row(i, m1, l1, m2, l2, acc, acc2);
        }
    }

    // ---- teardown: all TMEM readers and the MMA issuer are done past this barrier
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
#undef BAR
}

// Combines the key ranges of a split forward, one thread per query row: with M = max_s m_s,
// l = sum_s l_s 2^(m_s - M) and acc likewise (acc is rescaled with m1, as in the recurrence);
// then the same finish as the unsplit kernel.  Ranges with no valid key for a row hold
// m = -1e30, l = acc = 0 and drop out (2^(m_s - M) = 0).
__global__ void __launch_bounds__(256)
streamkl_splitk_merge_kernel(const float* __restrict__ part, int splits, long long R, float scale,
                             float* __restrict__ kl, float* __restrict__ lse1, float* __restrict__ lse2) {
    // launched as a programmatic dependent of the forward: wait until that grid has completed
    // and its partial states are visible (no-op when launched without the dependency)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (long long o = blockIdx.x * (long long)blockDim.x + threadIdx.x; o < R;
         o += (long long)gridDim.x * blockDim.x) {
        float M1 = -1e30f, M2 = -1e30f;
        for (int s = 0; s < splits; ++s) {
            M1 = fmaxf(M1, part[(s * 5 + 0) * R + o]);
            M2 = fmaxf(M2, part[(s * 5 + 2) * R + o]);
        }
        float L1 = 0.f, L2 = 0.f, A = 0.f;
        for (int s = 0; s < splits; ++s) {
            const float* q = part + s * 5 * R + o;
            const float a1 = ex2(q[0] - M1);
            const float a2 = ex2(q[2 * R] - M2);
            L1 = fmaf(q[R], a1, L1);
            A = fmaf(q[4 * R], a1, A);
            L2 = fmaf(q[3 * R], a2, L2);
        }
        const float LN2 = 0.6931471805599453f;
        const float lg1 = log2f(L1);
        const float lg2 = log2f(L2);
        lse1[o] = (M1 + lg1) * LN2;
        lse2[o] = (M2 + lg2) * LN2;
        kl[o] = scale * A / L1 + ((M2 - M1) + (lg2 - lg1)) * LN2;
    }
}

}  // namespace skl
