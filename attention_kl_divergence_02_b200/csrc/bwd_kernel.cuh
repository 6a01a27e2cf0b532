// bwd_kernel.cuh -- StreamKL backward on sm_100a.
//
// Gradient of sum_i g_i KL_i with one distribution held fixed (StreamKL technical summary,
// gist.science, Portuguese, "2. Estratégia de Recomputação (Passagem Backward)"):
//   mode 1 (P1 fixed):  dS2 = g * (P2 - P1)                         -> dQ2, dK2
//   mode 2 (P2 fixed):  dS1 = g * P1 * ((S1-LSE1) - (S2-LSE2) - KL) -> dQ1, dK1
// with P_t = exp(S_t - LSE_t) regenerated tile by tile from the saved LSEs ("Regeneração")
// and the mode-2 log-ratio taken from logit differences, never log P ("Estabilidade
// Numérica").  dQ = scale * dS K, dK = scale * dS^T Q.
//
// One CTA owns one 128-row query tile of one (batch, query head): Q1, Q2 and the rows'
// saved statistics stay on chip while the key tiles the rows can see (causal: up to the
// diagonal) stream through a ring of shared-memory slots, so each (query tile, key tile)
// pair is visited exactly once ("Fusão de Kernel").  Per visit n:
//   tensor core : S1 = Q1 K1^T, S2 = Q2 K2^T               (TMEM, lane = query row)
//   4 compute warpgroups: dS for 32 key columns each (thread = query row: the row's LSEs,
//                 KL and g sit in registers for the CTA's whole life) -> bf16, written
//                 once into one of two swizzled shared tiles [query][key] (visit parity)
//                 that feed both MMAs below
//   tensor core : dQ += dS K_free    (dS read K-major; TMEM accumulator over all visits:
//                                     dQ never leaves the chip until the end)
//                 dKp  = dS^T Q_free (dS read MN-major; TMEM, lane = key)
//   flush warpgroup: dKp from TMEM into registers, then into an fp32 dK workspace with
//                 16-byte vector reductions in L2 (red.global.add.v4.f32)
// Streaming the key tile (32 KiB with shared keys) instead of the query pair keeps the
// per-visit load small enough for a ring that prefetches two visits ahead; the MMA issuer
// looks one visit ahead (S of visit n+1 runs while the warpgroups turn S of visit n into
// dS), and the two dS tiles let the warpgroups write dS of visit n+1 while the dQ and dK
// MMAs of visit n still read theirs, so the tensor core is handed work without waiting for
// the write.
//
// At d = 64, when a KV group has an even number of query heads (HP = 2), a CTA owns the same
// query tile of two heads of the group: visits alternate between the heads for each key tile
// (loaded once), each head's dQ has its own TMEM columns, and the dK partial of a key tile
// sums both heads' visits before one flush.
//
// When the query tiles alone would leave SMs idle, the library splits each tile's key tiles
// into ranges (one CTA each); dQ is then added into a second tile-blocked fp32 workspace
// instead of being written once, and converted like dK.
//
// The workspace is private to the library and tile-blocked: one contiguous 128 x d block
// per (batch, KV head, key tile), laid out [lane quarter][32-column chunk][4-column group]
// [lane][4], the order in which the flush warps hold it; the convert kernel turns it into
// row-major bf16 dK.
//
// Roles (704 threads): warps 0-3 = dK flush warpgroup, warps 4..19 = four compute
// warpgroups, warp 20 = TMA producer, warp 21 = TMEM allocator + MMA issuer.  Warp w may
// touch TMEM lanes 32*(w%4)..+31, which is why each 128-lane reader is a group of four
// consecutive warps starting at a multiple of four.
#pragma once

#include "sm100.cuh"

namespace skl {

struct BwdParams {
    int B, Hq, Hkv, NQ, NK;
    int causal;
    int nkt;        // key tiles per (b, KV head)
    int nqt;        // query tiles per head
    float sl2;      // scale * log2(e)
    float scale;
    const float* kl;
    const float* lse1;
    const float* lse2;
    const float* dkl;
    float* dk_ws;   // fp32, tile-blocked (see above)
    uint16_t* dq;   // bf16 [B,Hq,NQ,d]
    int splits;     // key ranges per query tile (1 = one CTA sees all of a tile's keys)
    int kps;        // key tiles per range
    float* dq_ws;   // splits > 1: fp32 dQ partial sums, tile-blocked like dk_ws (planes B*Hq)
};

constexpr int kBwdThreads = 704;
constexpr int kBwdWG = 4;          // compute warpgroups
constexpr int kBwdComputeWarp0 = 4;
constexpr int kBwdProducerWarp = 20;
constexpr int kBwdMmaWarp = 21;
constexpr int kBwdHeadGroup = 2;   // (batch, head) planes scheduled together

// HP = query heads per CTA (1, or 2 at d = 64 when a KV group has an even number of query
// heads: the CTA then owns the same query tile of two heads that share their keys, visits
// every key tile once per head, and the dK partial of a key tile sums both heads' visits in
// TMEM before it is reduced).
template <int D, bool SHARED_K, int HP = 1>
struct BwdCfg {
    static_assert(HP == 1 || (HP == 2 && D == 64), "two heads per CTA only at d = 64");
    static constexpr int kTile = 128 * D * 2;                      // one 128-row bf16 tile
    static constexpr int kBoxes = D / 64;
    static constexpr int kBox = 128 * 128;
    static constexpr int kPerVisit = SHARED_K ? 1 : 2;             // key tiles streamed per key step
    static constexpr int kSlots = (D == 128) ? 3 : (HP == 2 ? 6 : 8);   // key-tile ring
    static constexpr int kQ1 = 0;                                  // head slot hs: + hs*kQStride
    static constexpr int kQ2 = kTile;
    static constexpr int kQStride = 2 * kTile;
    static constexpr int kRing = HP * 2 * kTile;                   // slot s at kRing + s*kTile
    static constexpr int kDS = kRing + kSlots * kTile;             // dS tiles, 2 x 128 x 128 bf16
    static constexpr int kDSBuf = 128 * 128 * 2;                   // dS tile b at kDS + b*kDSBuf
    static constexpr int kBar = kDS + 2 * kDSBuf;
    static constexpr int Q_FULL = 0;
    static constexpr int K_FULL = 1;                // + s
    static constexpr int K_EMPTY = 1 + kSlots;      // + s
    static constexpr int S_FULL = 1 + 2 * kSlots;
    static constexpr int S_FREE = S_FULL + 1;
    // DS_FULL + b: dS tile b written by the compute warps AND the dK columns of the
    // previous visit read out by the flush warps -- the one wait before dQ and dK
    static constexpr int DS_FULL = S_FULL + 2;      // + b
    static constexpr int DS_FREE = S_FULL + 4;      // + b
    static constexpr int DK_FULL = S_FULL + 6;
    static constexpr int DQ_DONE = S_FULL + 7;
    static constexpr int DONE = S_FULL + 8;
    static constexpr int kNumBars = DONE + 1;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kSmem = kMisc + 16 + 1024;
    // dQ of head slot hs at kColDQ + hs*D (HP = 2 only at d = 64: columns 256..383)
    static constexpr uint32_t kColS1 = 0, kColS2 = 128, kColDQ = 256, kColDK = 384;
};

// Visit n of a CTA -> key tile.  The CTA owns key tiles [lo, hi): range `sp` of kps tiles,
// clipped to the tiles its rows can see (causal: up to the diagonal tile qt).  Causal: from
// the diagonal end downwards.  Non-causal: rotated by query tile and head so that CTAs
// working at the same time reduce into different dK blocks.  count may be 0 (a range past
// the diagonal).
struct BwdSchedule {
    int lo, hi, rot, causal, count;
    __device__ BwdSchedule(const BwdParams& p, int qt_, int h, int sp) {
        causal = p.causal;
        lo = sp * p.kps;
        int end = min(p.nkt, lo + p.kps);
        if (causal) end = min(end, qt_ + 1);
        hi = end;
        count = max(0, end - lo);
        rot = count > 0 ? (qt_ + h) % count : 0;
    }
    __device__ int key_tile(int n) const {
        if (causal) return hi - 1 - n;
        const int u = n + rot;
        return lo + (u >= count ? u - count : u);
    }
};

// p[0..3] += (a, b, c, d) in L2, one 16-byte fp32 vector reduction (p 16-byte aligned).
__device__ __forceinline__ void red_add_v4(float* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(__uint_as_float(a)),
                 "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Which of a chunk's four column pairs take their P2 exponential on the FMA pipe instead of
// the exponential unit (mode 1 only; mode 2 has one exponential per element and leaves the
// unit half idle).  Two of the chunk's eight exponential pairs = a quarter of the mode-1
// exponentials.
#ifndef SKL_BWD_EMU2
#define SKL_BWD_EMU2 0x5
#endif

// dS of one query row over 8 key columns, packed to 4 bf16 pairs.  x = S1 raw, y = S2 raw;
// a = LSE1*log2(e); b = LSE2*log2(e) (mode 1) or LSE2-LSE1-KL (mode 2); g = upstream
// gradient.  FOLDED: g >= 0 has been folded into the exponents (a and, in mode 1, b
// lowered by log2 g, so 2^(u - a) is already g*P) and g is not multiplied again.  Adjacent
// columns are processed as fp32x2 pairs.  With MASKED, columns k >= lim are zero.
template <int MODE, bool MASKED, bool FOLDED>
__device__ __forceinline__ void ds_chunk(const uint32_t (&xa)[8], const uint32_t (&ya)[8],
                                         float sl2, float scale, float a, float b, float g,
                                         int lim, uint32_t* packed) {
    const float2 sl = make_float2(sl2, sl2);
    const float2 na = make_float2(-a, -a);
    const float2 nb = make_float2(-b, -b);
    const float2 bb = make_float2(b, b);
    const float2 gg = make_float2(g, g);
    const float2 sc = make_float2(scale, scale);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
        const float2 xk = make_float2(__uint_as_float(xa[2 * pr]), __uint_as_float(xa[2 * pr + 1]));
        const float2 yk = make_float2(__uint_as_float(ya[2 * pr]), __uint_as_float(ya[2 * pr + 1]));
        const float2 u1 = __ffma2_rn(xk, sl, na);
        const float2 p1 = make_float2(ex2(u1.x), ex2(u1.y));
        float2 v;
        if (MODE == 1) {
            const float2 u2 = __ffma2_rn(yk, sl, nb);
            const float2 p2 = ((SKL_BWD_EMU2 >> pr) & 1) ? ex2_poly2(u2)
                                                         : make_float2(ex2(u2.x), ex2(u2.y));
            v = __ffma2_rn(p1, neg1, p2);                  // (g)P2 - (g)P1
            if (!FOLDED) v = __fmul2_rn(v, gg);
        } else {
            const float2 r = __ffma2_rn(__ffma2_rn(yk, neg1, xk), sc, bb);   // scale(x-y) + b
            v = __fmul2_rn(p1, r);
            if (!FOLDED) v = __fmul2_rn(v, gg);
        }
        if (MASKED) {
            if (2 * pr >= lim) v.x = 0.f;
            if (2 * pr + 1 >= lim) v.y = 0.f;
        }
        packed[pr] = pack_bf16(v.x, v.y);
    }
}

template <int MODE>
__device__ __forceinline__ void ds_chunk_any(bool masked, bool folded, const uint32_t (&xa)[8],
                                             const uint32_t (&ya)[8], float sl2, float scale,
                                             float a, float b, float g, int lim, uint32_t* packed) {
    if (folded) {
        if (masked) ds_chunk<MODE, true, true>(xa, ya, sl2, scale, a, b, g, lim, packed);
        else ds_chunk<MODE, false, true>(xa, ya, sl2, scale, a, b, g, 8, packed);
    } else {
        if (masked) ds_chunk<MODE, true, false>(xa, ya, sl2, scale, a, b, g, lim, packed);
        else ds_chunk<MODE, false, false>(xa, ya, sl2, scale, a, b, g, 8, packed);
    }
}

template <int D, bool SHARED_K, int MODE, int HP>
__global__ void __launch_bounds__(kBwdThreads, 1)
streamkl_bwd_kernel(const __grid_constant__ CUtensorMap tmQ1, const __grid_constant__ CUtensorMap tmQ2,
                    const __grid_constant__ CUtensorMap tmK1, const __grid_constant__ CUtensorMap tmK2,
                    const BwdParams p) {
    using C = BwdCfg<D, SHARED_K, HP>;
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

    // ---- work unit.  The (batch, head) planes are taken kBwdHeadGroup at a time, and
    // within a group the heaviest causal query tiles are handed out first.  The CTAs in
    // flight then reduce into the dK blocks of a few KV heads only (a few MB per head), so
    // the partial sums meet in L2 instead of going back and forth to DRAM (a group of 2
    // measured best of 2, 4, 8 and 16 on the causal and GQA workloads).
    // With key ranges (few query tiles, many keys), the ranges of one query tile are
    // neighbours in the grid.  With HP = 2 a "plane" is a pair of query heads (h, h+1) of one
    // KV group.
    const int HU = p.Hq / HP;                 // head units per batch
    const int BH = p.B * HU;
    const int sp = blockIdx.x % p.splits;
    const int ub = blockIdx.x / p.splits;
    const int per_group = kBwdHeadGroup * p.nqt;
    const int group = ub / per_group;
    const int gh = min(kBwdHeadGroup, BH - group * kBwdHeadGroup);   // planes in this group
    const int r_in = ub - group * per_group;
    const int unit = r_in / gh;
    const int bhu = group * kBwdHeadGroup + r_in % gh;
    const int qt = p.causal ? (p.nqt - 1 - unit) : unit;
    const int b = bhu / HU;
    const int h = (bhu % HU) * HP;            // first query head of the unit
    const int bh = b * p.Hq + h;              // its (batch, head) plane; head slot hs is bh + hs
    const int bhk = b * p.Hkv + h / (p.Hq / p.Hkv);
    const int q0 = qt * 128;
    const BwdSchedule sched(p, qt, h, sp);
    const int N = sched.count;                // key steps; visit v = key step v / HP, head slot v % HP
    const int V = N * HP;
    constexpr bool mode1 = (MODE == 1);
    // Key tiles of a visit enter the ring in the order (fixed distribution's, free
    // distribution's): j = 0 is released as soon as S is done, j = 1 after dQ.  With three
    // slots, the look-ahead S(n+1) then lands in slots that S(n) and dQ(n-1) have freed.
    // (With shared keys there is one tile per visit, j = 0, released after dQ.)
    auto ring_idx = [](int n, int j) { return n * C::kPerVisit + j; };
    // j of K1 and of K2; the free distribution is (Q2, K2) in mode 1, (Q1, K1) in mode 2
    constexpr int kJ1 = SHARED_K ? 0 : (mode1 ? 0 : 1);
    constexpr int kJ2 = SHARED_K ? 0 : (mode1 ? 1 : 0);
    constexpr int kJFree = SHARED_K ? 0 : 1;
    const uint32_t qfree = sb + (mode1 ? C::kQ2 : C::kQ1);   // head slot hs: + hs*kQStride

    if (threadIdx.x == 0) {
        mbar_init(BAR(C::Q_FULL), 1);
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(BAR(C::K_FULL + s), 1);
            mbar_init(BAR(C::K_EMPTY + s), 1);
        }
        mbar_init(BAR(C::S_FULL), 1);
        mbar_init(BAR(C::S_FREE), 32 * 4 * kBwdWG);
        // the flush warps' "dK read out" arrival gates the visits that start a key step's dK:
        // every visit when HP = 1, the even ones (tile 0) when HP = 2
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(C::DS_FULL + b), 32 * 4 * kBwdWG + ((HP == 1 || b == 0) ? 128 : 0));
            mbar_init(BAR(C::DS_FREE + b), 1);
        }
        mbar_init(BAR(C::DK_FULL), 1);
        mbar_init(BAR(C::DQ_DONE), 1);
        mbar_init(BAR(C::DONE), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == kBwdProducerWarp) {
        // ================================================================ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ1);
            tma_prefetch_desc(&tmQ2);
            tma_prefetch_desc(&tmK1);
            if (!SHARED_K) tma_prefetch_desc(&tmK2);
            mbar_arrive_expect_tx(BAR(C::Q_FULL), HP * 2 * C::kTile);
            for (int hs = 0; hs < HP; ++hs)
                for (int bx = 0; bx < C::kBoxes; ++bx) {
                    tma_load_3d(sb + C::kQ1 + hs * C::kQStride + bx * C::kBox, &tmQ1, BAR(C::Q_FULL),
                                bx * 64, q0, bh + hs);
                    tma_load_3d(sb + C::kQ2 + hs * C::kQStride + bx * C::kBox, &tmQ2, BAR(C::Q_FULL),
                                bx * 64, q0, bh + hs);
                }
            uint32_t it = 0;
            bool ok = true;
            for (int n = 0; n < N && ok; ++n) {
                const int kt = sched.key_tile(n);
#pragma unroll
                for (int j = 0; j < C::kPerVisit; ++j) {
                    const uint32_t s = it % C::kSlots;
                    const uint32_t u = it / C::kSlots;
                    if (u > 0 && !mbar_wait(BAR(C::K_EMPTY + s), (u - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(BAR(C::K_FULL + s), C::kTile);
                    const CUtensorMap* map = (j == kJ1) ? &tmK1 : &tmK2;
                    for (int bx = 0; bx < C::kBoxes; ++bx)
                        tma_load_3d(sb + C::kRing + s * C::kTile + bx * C::kBox, map,
                                    BAR(C::K_FULL + s), bx * 64, kt * 128, bhk);
                    ++it;
                }
            }
            // drain every copy started here
            drain_wait(BAR(C::Q_FULL), 0);
            for (uint32_t s = 0; s < (uint32_t)C::kSlots; ++s) {
                if (it > s) {
                    const uint32_t fills = (it - s - 1) / C::kSlots + 1;
                    drain_wait(BAR(C::K_FULL + s), (fills - 1) & 1);
                }
            }
        }
    } else if (warp == kBwdMmaWarp) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);   // Q, K both K-major
            constexpr uint32_t idQ = idesc_bf16(128, D, 0, 1);     // dS K-major, K MN-major
            constexpr uint32_t idK = idesc_bf16(128, D, 1, 1);     // dS^T MN-major, Q MN-major
            auto slot_of = [&](int n, int j) { return (uint32_t)(ring_idx(n, j) % C::kSlots); };
            auto fill_parity = [&](int n, int j) { return (uint32_t)((ring_idx(n, j) / C::kSlots) & 1); };
            // Descriptors are built once per operand base and advanced by the operand's byte
            // offset / 16 (the 14-bit start-address field cannot carry: shared addresses stay
            // below 2^18 and every offset is a multiple of 16), so the issuing thread spends
            // about one instruction per descriptor between MMAs; those of the resident query
            // tiles are loop-invariant.
            auto dadd = [](uint64_t dsc, uint32_t bytes) { return dsc + (uint64_t)(bytes >> 4); };
            const uint64_t dq1k = sw128_desc(sb + C::kQ1, 16, 1024);        // Q1, K-major
            const uint64_t dq2k = sw128_desc(sb + C::kQ2, 16, 1024);        // Q2, K-major
            const uint64_t dqfm = sw128_desc(qfree, C::kBox, 1024);         // Q_free, MN-major
            constexpr uint32_t kQS = (uint32_t)C::kQStride;                  // next head slot's Q
            // S of visit v (key step v / HP, head slot v % HP); returns false if a wait gave up
            auto issue_S = [&](int v) -> bool {
                const int n = v / HP;
                const uint32_t qo = (uint32_t)(v % HP) * kQS;
                const uint32_t s1 = slot_of(n, kJ1);
                const uint32_t s2 = SHARED_K ? s1 : slot_of(n, kJ2);
                if (!mbar_wait(BAR(C::K_FULL + s1), fill_parity(n, kJ1), abort_flag)) return false;
                if (!SHARED_K && !mbar_wait(BAR(C::K_FULL + s2), fill_parity(n, kJ2), abort_flag))
                    return false;
                tc_fence_after();
                const uint64_t dk1 = sw128_desc(sb + C::kRing + s1 * C::kTile, 16, 1024);
                const uint64_t dk2 = SHARED_K ? dk1 : sw128_desc(sb + C::kRing + s2 * C::kTile, 16, 1024);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * C::kBox + (k & 3) * 32;
                    mma_bf16_ss(tmem + C::kColS1, dadd(dq1k, qo + off), dadd(dk1, off), idS, k > 0);
                }
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * C::kBox + (k & 3) * 32;
                    mma_bf16_ss(tmem + C::kColS2, dadd(dq2k, qo + off), dadd(dk2, off), idS, k > 0);
                }
                mma_commit(BAR(C::S_FULL));
                // with distinct keys, the fixed distribution's key tile (j = 0) is done after the
                // key step's last S
                if (!SHARED_K && v % HP == HP - 1) mma_commit(BAR(C::K_EMPTY + slot_of(n, 0)));
                return true;
            };
            // dQ of visit m, once its dS tile is written (and the flush has read the dK of the
            // previous key step, when m starts one)
            auto issue_dq = [&](int m) -> bool {
                const int n = m / HP;
                const int hs = m % HP;
                const uint32_t ds = sb + C::kDS + (m & 1) * C::kDSBuf;
                const uint64_t ddsk = sw128_desc(ds, 16, 1024);         // dS, K-major (A of dQ)
                const uint64_t dkfm = sw128_desc(sb + C::kRing + slot_of(n, kJFree) * C::kTile,
                                                 C::kBox, 1024);        // K_free, MN-major
                if (!mbar_wait(BAR(C::DS_FULL + (m & 1)), (m >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                // dQ of head slot hs += dS K_free, accumulated over every visit of that slot
#pragma unroll
                for (int k = 0; k < 8; ++k) {   // 128 keys, 16 per MMA
                    mma_bf16_ss(tmem + C::kColDQ + (uint32_t)(hs * D),
                                dadd(ddsk, (k >> 2) * C::kBox + (k & 3) * 32),
                                dadd(dkfm, k * 2048), idQ, (m >= HP || k > 0));
                }
                if (hs == HP - 1) mma_commit(BAR(C::K_EMPTY + slot_of(n, kJFree)));
                return true;
            };
            // dK partial of visit m: dS^T Q_free of its head slot, fresh at a key step's first
            // visit and accumulated over the others; frees its dS tile
            auto issue_dk = [&](int m) {
                const int hs = m % HP;
                const uint64_t ddsm = sw128_desc(sb + C::kDS + (m & 1) * C::kDSBuf, C::kBox, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {   // 128 queries, 16 per MMA
                    mma_bf16_ss(tmem + C::kColDK, dadd(ddsm, k * 2048),
                                dadd(dqfm, (uint32_t)hs * kQS + k * 2048), idK, (hs > 0 || k > 0));
                }
                if (hs == HP - 1) mma_commit(BAR(C::DK_FULL));
                mma_commit(BAR(C::DS_FREE + (m & 1)));
            };
            bool ok = mbar_wait(BAR(C::Q_FULL), 0, abort_flag);
            if (ok && V > 0) ok = issue_S(0);
            if constexpr (D == 64) {
            // Issue order dQ(n-1), S(n+1), dK(n-1): the tensor core executes in issue order, so
            // S(n+1) -- which the compute warps wait for -- queues behind 8 dQ MMAs instead of
            // 16 dQ and dK MMAs.  dQ(n-1) still frees visit n-1's key slot before S(n+1); the
            // two dS tiles cover the later dK.  Measured faster at d = 64 (GQA, mode 1: 6.83 ->
            // 6.4 ms), slower at d = 128 (headline 4.33 -> 4.8 ms), so d = 128 keeps the order
            // S(n+1), dQ(n), dK(n).
            for (int v = 0; v <= V && ok; ++v) {
                if (v >= 1 && !issue_dq(v - 1)) break;
                if (v + 1 < V) {
                    if (!mbar_wait(BAR(C::S_FREE), v & 1, abort_flag)) break;
                    tc_fence_after();
                    if (!issue_S(v + 1)) break;
                }
                if (v >= 1) issue_dk(v - 1);
            }
            } else {
            for (int v = 0; v < V && ok; ++v) {
                if (v + 1 < V) {
                    if (!mbar_wait(BAR(C::S_FREE), v & 1, abort_flag)) break;
                    tc_fence_after();
                    if (!issue_S(v + 1)) break;
                }
                if (!issue_dq(v)) break;
                issue_dk(v);
            }
            }
            mma_commit(BAR(C::DQ_DONE));
            mma_commit(BAR(C::DONE));
            drain_wait(BAR(C::DONE), 0);
        }
    } else if (warp < kBwdComputeWarp0) {
        // ================================================================ dK flush warpgroup
        const int quarter = warp;               // TMEM lanes 32*quarter.. = key rows
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        mbar_arrive(BAR(C::DS_FULL));               // visit 0 has no earlier dK to wait for
        for (int n = 0; n < N; ++n) {               // one dK partial per key step
            const int kt = sched.key_tile(n);
            if (!mbar_wait(BAR(C::DK_FULL), n & 1, abort_flag)) break;
            tc_fence_after();
            // this lane's 16-byte groups of its key row: [chunk][group][lane][4] in the block
            float* dst = p.dk_ws + ((size_t)bhk * p.nkt + kt) * (128 * D) + (size_t)quarter * (32 * D) +
                         lane * 4;
#pragma unroll 1
            for (int c = 0; c < D / 32; c += 2) {
                uint32_t v[2][32];
                tmem_ld32(lane_base + C::kColDK + c * 32, v[0]);
                tmem_ld32(lane_base + C::kColDK + c * 32 + 32, v[1]);
                tmem_wait_ld();
                if (c + 2 == D / 32) {           // the dK columns are all in registers: the
                    tc_fence_before();           // next key step's first visit may overwrite them
                    mbar_arrive(BAR(C::DS_FULL + (((n + 1) * HP) & 1)));
                }
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        red_add_v4(dst + (c + h) * (32 * 32) + g * 128, v[h][4 * g], v[h][4 * g + 1],
                                   v[h][4 * g + 2], v[h][4 * g + 3]);
            }
        }
    } else if (warp < kBwdComputeWarp0 + 4 * kBwdWG) {
        // ================================================================ compute warpgroups
        const int wg = (warp - kBwdComputeWarp0) >> 2;   // key columns [32*wg, 32*wg + 32)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;      // TMEM lane = query row
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sl2 = p.sl2;
        const float scale = p.scale;
        const float LOG2E = 1.4426950408889634f;
        // this thread's 64 bytes of dS row r in tile 0: box (wg/2), 16-byte chunks 4*(wg&1)..+3
        uint8_t* ds_row0 = smem + C::kDS + (wg >> 1) * C::kBox + r * 128;
        const int q = q0 + r;
        // this row's statistics in each head slot, for the CTA's whole life: a = LSE1*log2(e),
        // bq = LSE2*log2(e) (mode 1) or LSE2 - LSE1 - KL (mode 2), g; rows past NQ get g = 0
        // (their dS is 0).  g is folded into the exponents when no row of the warp has g < 0;
        // a row with g = 0 (or past NQ) has dS = 0 exactly: it takes the masked variant with
        // every column masked (folding log2 0 = -inf would leave 2^-126 where the FMA-pipe
        // exponential clamps its argument)
        float a_[HP], bq_[HP], g_[HP];
        bool folded_[HP], zero_[HP];
#pragma unroll
        for (int hs = 0; hs < HP; ++hs) {
            float a = 0.f, bq = 0.f, g = 0.f;
            if (q < p.NQ) {
                const size_t o = (size_t)(bh + hs) * p.NQ + q;
                const float L1 = p.lse1[o], L2 = p.lse2[o];
                a = L1 * LOG2E;
                bq = mode1 ? L2 * LOG2E : (L2 - L1 - p.kl[o]);
                g = p.dkl[o];
            }
            const bool folded = !__any_sync(0xffffffffu, g < 0.f);
            if (folded && g > 0.f) {
                const float lg = log2f(g);
                a -= lg;
                if (mode1) bq -= lg;
            }
            a_[hs] = a;
            bq_[hs] = bq;
            g_[hs] = g;
            folded_[hs] = folded;
            zero_[hs] = !(g != 0.f);
        }
        const int kc0 = wg * 32;
        bool ok = true;
        for (int v = 0; v < V; ++v) {
            const int n = v / HP;
            const bool h1 = HP == 2 && (v & 1);   // head slot 1 (constant-index selects)
            const float a = h1 ? a_[HP - 1] : a_[0];
            const float bq = h1 ? bq_[HP - 1] : bq_[0];
            const float g = h1 ? g_[HP - 1] : g_[0];
            const bool folded = h1 ? folded_[HP - 1] : folded_[0];
            const bool zero_row = h1 ? zero_[HP - 1] : zero_[0];
            const int kt = sched.key_tile(n);
            const int k0 = kt * 128;
            // masked columns: keys past the diagonal of a causal diagonal tile, and
            // zero-filled keys past NK; columns k < lim of this warpgroup are valid
            bool need_mask = (p.causal && kt == qt) || (k0 + 128 > p.NK);
            int lim = 32;
            if (need_mask) {
                lim = min(lim, p.NK - k0 - kc0);
                if (p.causal && kt == qt) lim = min(lim, r - kc0 + 1);
            }
            if (zero_row) {
                need_mask = true;
                lim = 0;
            }
            if (!mbar_wait(BAR(C::S_FULL), v & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // the warpgroup's 32 columns in four 8-column chunks: the load of chunk c+1 is in
            // flight while chunk c is turned into dS, so only the first load's latency shows
            uint32_t packed[16];
            uint32_t xa[2][8], ya[2][8];
            tmem_ld8(lane_base + C::kColS1 + kc0, xa[0]);
            tmem_ld8(lane_base + C::kColS2 + kc0, ya[0]);
            tmem_wait_ld_regs(xa[0], ya[0]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (c < 3) {
                    tmem_ld8(lane_base + C::kColS1 + kc0 + 8 * (c + 1), xa[(c + 1) & 1]);
                    tmem_ld8(lane_base + C::kColS2 + kc0 + 8 * (c + 1), ya[(c + 1) & 1]);
                }
                ds_chunk_any<MODE>(need_mask, folded, xa[c & 1], ya[c & 1], sl2, scale, a, bq, g,
                                   lim - 8 * c, packed + 4 * c);
                if (c < 3) tmem_wait_ld_regs(xa[(c + 1) & 1], ya[(c + 1) & 1]);
                if (c == 2) {
                    tc_fence_before();
                    mbar_arrive(BAR(C::S_FREE));  // all of this thread's S columns are read
                }
            }
            // dS tile v&1 was last read by the MMAs of visit v-2
            if (v > 1 && !mbar_wait(BAR(C::DS_FREE + (v & 1)), ((v >> 1) - 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            uint8_t* ds_row = ds_row0 + (v & 1) * C::kDSBuf;
            const int cbase = (wg & 1) * 4;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int phys = (cbase + c) ^ (r & 7);
                *reinterpret_cast<uint4*>(ds_row + phys * 16) =
                    make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
            }
            fence_async_smem();
            mbar_arrive(BAR(C::DS_FULL + (v & 1)));
        }
        // dQ of this query tile, accumulated over every visit of the CTA.  One key range:
        // scale, round, store.  Several: add it into the fp32 dQ workspace (the convert kernel
        // scales and rounds once every range has added its part).
        if (ok && N > 0 && mbar_wait(BAR(C::DQ_DONE), 0, abort_flag)) {
            tc_fence_after();
#pragma unroll 1
            for (int hs = 0; hs < HP; ++hs) {
            constexpr int kCols = D / 4;          // dQ columns per warpgroup
            uint32_t v[kCols];
            if constexpr (D == 128) {
                tmem_ld32(lane_base + C::kColDQ + wg * kCols, v);
            } else {
                tmem_ld16(lane_base + C::kColDQ + hs * D + wg * kCols, v);
            }
            tmem_wait_ld();
            if (p.splits > 1) {
                // tile-blocked: [quarter][32-column chunk][4-column group][lane][4]
                float* blk = p.dq_ws + ((size_t)(bh + hs) * p.nqt + qt) * (128 * D) +
                             (size_t)quarter * (32 * D) + lane * 4;
                const int c = (wg * kCols) / 32;          // chunk of this warpgroup's columns
                const int g0 = ((wg * kCols) % 32) / 4;   // first 4-column group in the chunk
#pragma unroll
                for (int g = 0; g < kCols / 4; ++g)
                    red_add_v4(blk + c * 1024 + (g0 + g) * 128, v[4 * g], v[4 * g + 1], v[4 * g + 2],
                               v[4 * g + 3]);
            } else if (q < p.NQ) {
                uint4* dst = reinterpret_cast<uint4*>(p.dq + ((size_t)(bh + hs) * p.NQ + q) * D +
                                                      wg * kCols);
#pragma unroll
                for (int k = 0; k < kCols / 8; ++k) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * k + e]) * scale;
                    dst[k] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]),
                                        pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
                }
            }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
#undef BAR
}

// out = bf16(scale * ws), un-blocking a tile-blocked fp32 workspace of `rows` rows per
// plane (planes = B*Hkv for dK) and ntiles 128-row tiles per plane.  One thread = one row's
// 32-column chunk: it reads 8 float4 (coalesced across the 32 lanes of the chunk) and
// writes 64 contiguous bytes of its row.
template <int D>
__global__ void __launch_bounds__(256)
streamkl_tile_convert_kernel(const float* __restrict__ ws, uint16_t* __restrict__ out, int planes,
                             int rows, int ntiles, float scale) {
    constexpr int kChunks = D / 32;
    const size_t total = (size_t)planes * ntiles * 128 * kChunks;   // (plane, tile, quarter, chunk, lane)
    for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < total;
         t += (size_t)gridDim.x * blockDim.x) {
        const int lane = (int)(t & 31);
        const size_t u = t >> 5;
        const int c = (int)(u % kChunks);
        const int quarter = (int)((u / kChunks) & 3);
        const size_t blk = u / kChunks / 4;        // plane * ntiles + tile
        const int tile = (int)(blk % ntiles);
        const size_t plane = blk / ntiles;
        const int row = tile * 128 + quarter * 32 + lane;
        if (row >= rows) continue;
        const float4* src = reinterpret_cast<const float4*>(
            ws + blk * (128 * D) + (size_t)(quarter * kChunks + c) * 1024) + lane;
        uint4* dst = reinterpret_cast<uint4*>(out + (plane * rows + row) * D + c * 32);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 a = src[(2 * k) * 32];
            const float4 e = src[(2 * k + 1) * 32];
            dst[k] = make_uint4(pack_bf16(a.x * scale, a.y * scale), pack_bf16(a.z * scale, a.w * scale),
                                pack_bf16(e.x * scale, e.y * scale), pack_bf16(e.z * scale, e.w * scale));
        }
    }
}

}  // namespace skl
