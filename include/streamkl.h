/*
 * streamkl.h -- C ABI of libstreamkl, a B200 (sm_100a) fused attention KL divergence.
 *
 * The operation ("StreamKL: Fast and Memory-Efficient KL Divergence for Boosting Attention
 * Distillation", abstract; StreamKL technical summary, gist.science, Portuguese,
 * "Definição do Problema"): for batch b, query head h and query row i,
 *
 *     s_t[j] = scale * <Q_t[b,h,i,:], K_t[b,h/(Hq/Hkv),j,:]>,   t = 1, 2
 *     P_t    = softmax of s_t over the valid keys (j < NK, and j <= i when causal)
 *     KL_i   = sum_j P1[j] * (log P1[j] - log P2[j])
 *
 * computed without ever forming P1 or P2 in memory.  Grouped query heads follow the GQA
 * definition of the KV-cache lecture notes (hackmd, "3. 架構層級的記憶體妥協").
 *
 * Conventions shared by every entry point:
 *  - Every pointer argument is a DEVICE pointer owned by the caller; the library keeps no
 *    reference after the call returns and allocates no device memory (its only device
 *    memory of its own is the static buffer of streamkl_bwd_noalloc and a status word).
 *  - Tensors are dense and row-major with the head dimension innermost:
 *      Q1, Q2, dQ : bf16 [B, Hq, NQ, d]        K1, K2, dK : bf16 [B, Hkv, NK, d]
 *      kl, lse1, lse2, dkl : fp32 [B, Hq, NQ]
 *    bf16 is IEEE-754 binary32 truncated to its upper 16 bits (passed as uint16_t).
 *  - Supported: d in {64, 128}; B, Hq, Hkv, NQ, NK >= 1; Hq % Hkv == 0; scale > 0 and
 *    finite; causal requires NQ == NK (the mask is j <= i); every pointer 16-byte aligned;
 *    B*Hq*NQ and B*Hkv*NK below 2^31 rows.  Anything else returns STREAMKL_ERR_UNSUPPORTED
 *    (shape or alignment outside the supported set) or STREAMKL_ERR_INVALID_ARG (null
 *    pointer, non-positive size, bad mode), and nothing is launched.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *    stream).  A return of STREAMKL_OK means the work was enqueued.  Errors that happen on
 *    the device later (a bounded pipeline wait that ran out) are recorded in a device status
 *    word that streamkl_device_status() reads.  On any error the outputs are undefined.
 *  - No call aborts the process or traps on the device.
 *  - K1 == K2 (the same pointer) means one shared key tensor: it is read once per tile.
 */
#ifndef STREAMKL_H
#define STREAMKL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    STREAMKL_OK = 0,
    STREAMKL_ERR_INVALID_ARG = 1,  /* null pointer, size < 1, mode not 1/2, workspace too small */
    STREAMKL_ERR_UNSUPPORTED = 2,  /* d not 64/128, Hq % Hkv, causal with NQ != NK, alignment */
    STREAMKL_ERR_CUDA = 3,         /* a CUDA runtime or driver call failed (launch, memset) */
    STREAMKL_ERR_TIMEOUT = 4       /* a kernel gave up on a pipeline wait (device status only) */
};

/*
 * Forward.  One pass over the key tiles per query row, keeping five running scalars per
 * row (m1, l1, m2, l2, acc) and returning KL = acc/l1 + LSE2 - LSE1 with
 * LSE_t = m_t + log l_t (StreamKL technical summary, "1. Formulação Online (Passagem
 * Forward)"; running sums rescaled by exp(m_old - m_new) when a maximum grows, as in the
 * FlashAttention lecture notes, hackmd, "4. Flash Attention 的核心數學重構").  Causal key
 * tiles past the diagonal are skipped entirely.
 *
 *   q1, k1, q2, k2 : bf16 inputs (see conventions); k1 == k2 selects the shared-key path.
 *   kl, lse1, lse2 : fp32 [B,Hq,NQ] outputs, overwritten; natural-log units.  These three
 *                    vectors are the whole saved state of the backward ("2. Estratégia de
 *                    Recomputação", "Estado Salvo").
 * Extra device memory: none.
 */
int streamkl_fwd(const uint16_t* q1, const uint16_t* k1, const uint16_t* q2, const uint16_t* k2,
                 int B, int Hq, int Hkv, int NQ, int NK, int d, float scale, int causal,
                 float* kl, float* lse1, float* lse2, void* stream);

/*
 * Both directions in one pass: KL(P1 || P2) and KL(P2 || P1) per query row, whose sum is the
 * symmetric (Jeffreys) divergence.  The pages only outline that fused online primitives
 * extend to other coupled two-distribution reductions (technical summary, "Significância");
 * this is the plainest such extension: the forward's five running scalars plus a sixth,
 * acc2 = sum_j exp(s2_j - m2) (s1_j - s2_j), rescaled like l2 whenever m2 grows, so that
 * KL(P2 || P1) = -acc2/l2 + LSE1 - LSE2.  The keys are read once for both directions.
 *
 *   kl12, kl21, lse1, lse2 : fp32 [B,Hq,NQ] outputs, overwritten (natural-log units).
 * Other arguments, errors and ownership as streamkl_fwd.  No key-range split (one CTA per query
 * block, or per head for at most 8 rows); extra device memory: none.
 */
int streamkl_fwd_sym(const uint16_t* q1, const uint16_t* k1, const uint16_t* q2, const uint16_t* k2,
                     int B, int Hq, int Hkv, int NQ, int NK, int d, float scale, int causal,
                     float* kl12, float* kl21, float* lse1, float* lse2, void* stream);

/*
 * Forward with the key tiles split into ranges, for few query rows and many keys (the
 * decoding case the technical summary's "3. Otimizações de Kernel de GPU" names for split-K):
 * each (query block, key range) is one CTA, so B*Hq*ceil(NQ/256) blocks that would leave
 * most of the 148 SMs idle become enough CTAs to stream the keys at HBM speed.  Every range
 * stores its rows' five running scalars; a second kernel merges the ranges exactly (each
 * rescaled to the common maximum, the online recurrence's own correction) and writes the
 * same outputs as streamkl_fwd.
 *
 *   splits    : number of key ranges; 0 = the library's choice (streamkl_fwd_splits).  A
 *               value above the number of 128-key tiles is reduced to it, and ranges are
 *               whole tiles, so fewer ranges than asked may be used.  1 = streamkl_fwd.
 *   workspace : device buffer of at least streamkl_fwd_splitk_workspace_bytes(B, Hq, NQ,
 *               NK, splits) bytes, 16-byte aligned, owned by the caller; its contents on
 *               entry do not matter.  May be NULL when that size is 0 (one range).
 * Other arguments, outputs, errors and ownership as streamkl_fwd.  Two kernels are launched
 * on `stream`; extra device memory: the workspace only.
 */
int streamkl_fwd_splitk(const uint16_t* q1, const uint16_t* k1, const uint16_t* q2,
                        const uint16_t* k2, int B, int Hq, int Hkv, int NQ, int NK, int d,
                        float scale, int causal, int splits, float* kl, float* lse1, float* lse2,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * The number of key ranges streamkl_fwd_splitk uses for splits = 0.  At most 8 query rows
 * (keys as the MMA's rows, two CTAs per SM): enough ranges for one wave of two CTAs per SM,
 * 1 when the heads alone fill it.  More rows: 1 when the query blocks alone fill the GPU,
 * else the fewest ranges within 3 % of the best of a waves x (tiles per range + 8) model, at
 * most 64.  Uses the current device's SM count.  Host-only; returns 1 for invalid sizes.
 */
int streamkl_fwd_splits(int B, int Hq, int NQ, int NK);

/*
 * Bytes of split-K workspace: 5 fp32 per query row per key range actually used (0 when only
 * one range is used, or for invalid sizes).  splits = 0 means the library's choice.
 */
size_t streamkl_fwd_splitk_workspace_bytes(int B, int Hq, int NQ, int NK, int splits);

/*
 * Bytes of fp32 workspace streamkl_bwd needs for these sizes: the dK accumulator,
 * B*Hkv*ceil(NK/128)*128*d*4 (whole 128-row key tiles), plus, when streamkl_bwd splits each
 * query tile's keys into ranges (its CTAs alone would leave SMs idle and there are at least
 * two key tiles), the dQ partial sums B*Hq*ceil(NQ/128)*128*d*4.  The backward runs one CTA
 * per query tile and query head, or per query tile and pair of query heads when d = 64 and
 * Hq/Hkv is even, so B*Hq*ceil(NQ/128) or half that CTAs before any split.  Returns 0 for
 * sizes outside the supported range.  The split decision depends on the SM count of the
 * current device (streamkl_num_sms), so query with the device current that the backward will
 * run on.
 */
size_t streamkl_bwd_workspace_bytes(int B, int Hq, int Hkv, int NQ, int NK, int d);

/*
 * Backward of sum_i dkl[i] * KL_i, recomputing P_t = exp(S_t - LSE_t) tile by tile from the
 * saved LSEs (technical summary, "2. Estratégia de Recomputação (Passagem Backward)",
 * "Regeneração").  With g = dkl:
 *   mode 1 (P1 fixed, "Configuração 1"): dS2 = g * (P2 - P1); outputs dQ2, dK2.
 *   mode 2 (P2 fixed, "Configuração 2"): dS1 = g * P1 * ((S1-LSE1) - (S2-LSE2) - KL),
 *        with the log-ratio taken from logit differences and the saved LSEs, never from
 *        log P ("Estabilidade Numérica"); outputs dQ1, dK1.
 *   dQ_t = scale * dS_t K_t,  dK_t = scale * dS_t^T Q_t summed over the query heads that
 *   share the KV head.  The fixed distribution gets no gradient; with k1 == k2 the
 *   returned dk is the gradient through the free distribution only.
 * One CTA owns a 128-row query tile and visits every key tile its rows see, once ("Fusão de
 * Kernel"); at d = 64 with an even number of query heads per KV head it owns that tile in two
 * heads of one group, and their dK partials meet on chip.  When those CTAs alone would leave
 * SMs idle (few query rows, long keys), each
 * tile's keys are split into ranges handled by separate CTAs and dQ is summed through the
 * workspace too; the choice is the library's and is reflected in
 * streamkl_bwd_workspace_bytes.  Launches: a workspace memset, the backward kernel, one
 * convert kernel for dK (and one for dQ when the keys are split).
 *
 *   kl, lse1, lse2 : the forward's outputs for the same inputs (read only).
 *   dkl            : fp32 [B,Hq,NQ] upstream gradient (read only).
 *   dq             : bf16 [B,Hq,NQ,d] output, overwritten.
 *   dk             : bf16 [B,Hkv,NK,d] output, overwritten.
 *   workspace      : caller-owned device buffer of at least
 *                    streamkl_bwd_workspace_bytes(B,Hq,Hkv,NQ,NK,d) bytes, 16-byte aligned; its
 *                    contents on entry do not matter and are undefined on exit.  Two calls
 *                    that run at the same time need two workspaces.
 */
int streamkl_bwd(int mode, const uint16_t* q1, const uint16_t* k1, const uint16_t* q2,
                 const uint16_t* k2, const float* kl, const float* lse1, const float* lse2,
                 const float* dkl, int B, int Hq, int Hkv, int NQ, int NK, int d, float scale,
                 int causal, uint16_t* dq, uint16_t* dk, void* workspace, size_t workspace_bytes,
                 void* stream);

/*
 * Size of the library's built-in backward scratch buffer (see streamkl_bwd_noalloc).
 */
#define STREAMKL_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * Backward that allocates nothing and takes no workspace argument.  This entry point has
 * no counterpart in the StreamKL papers; it exists for callers that may not allocate
 * device memory at all -- for example code running inside a framework whose allocator
 * owns all of the GPU's memory and forbids side allocations, a service whose device-memory
 * budget is fixed once it has started, or a latency-critical path that cannot afford the
 * device-wide synchronisation that cudaMalloc/cudaFree can cause.
 *
 * Same arguments, semantics and outputs as streamkl_bwd, minus workspace/workspace_bytes:
 * what streamkl_bwd keeps in its workspace -- the fp32 dK accumulator, plus the fp32 dQ
 * partial sums when the key-range split is chosen -- lives in a fixed
 * STREAMKL_NOALLOC_SCRATCH_BYTES (32 MiB) buffer compiled into the library as a static
 * device array.  Every GPU on which the library is loaded holds that buffer until the
 * process exits.
 *  - The limit: streamkl_bwd_workspace_bytes(B, Hq, Hkv, NQ, NK, d) <= 32 MiB (for example
 *    at most 4 KV heads of 16384 keys at d = 128).  Larger sizes return
 *    STREAMKL_ERR_UNSUPPORTED and launch nothing; use streamkl_bwd for those.
 *  - The first call on each device looks up the buffer's device address (a set-up done
 *    with that device current, repeated only if the device's context has changed since,
 *    e.g. after cudaDeviceReset); make that first call before any stream capture begins on
 *    the device.
 *  - All calls on a device share the one buffer; it is cleared at the start of every call,
 *    so leftover contents do not matter, but two calls that can run at the same time on
 *    the GPU (different streams, no ordering between them) race on it and give undefined
 *    results.  Order such calls on one stream or with events.
 */
int streamkl_bwd_noalloc(int mode, const uint16_t* q1, const uint16_t* k1, const uint16_t* q2,
                         const uint16_t* k2, const float* kl, const float* lse1, const float* lse2,
                         const float* dkl, int B, int Hq, int Hkv, int NQ, int NK, int d,
                         float scale, int causal, uint16_t* dq, uint16_t* dk, void* stream);

/*
 * Throughput probe of the two exponential paths the kernels use; no part of the KL
 * computation.  The forward spends two exponentials per (row, key) pair with no second GEMM
 * to amortise them (technical summary, "1. Formulação Online"), so their rate, not the
 * tensor core, is its floor; this measures that rate.
 *   kind 0: ex2.approx on the exponential unit (MUFU); kind 1: the FMA-pipe polynomial
 *           the kernels evaluate part of their exponentials with.
 *   iters : loop trips per thread (>= 1); the run takes about iters * 3 us (kind 0).
 *   n_exp : if not NULL, receives the number of exponentials the launch evaluates
 *           (4 CTAs per SM x 256 threads x 8 independent chains x iters).
 * One kernel is launched on `stream`; the caller times it (CUDA events) and divides.
 * Reads and writes no memory.  Returns STREAMKL_ERR_INVALID_ARG for a bad kind or iters.
 */
int streamkl_probe_exp2(int kind, int iters, long long* n_exp, void* stream);

/*
 * SM count of the current device, which the library's grid-sizing choices (key ranges of
 * the split-K forward and of the backward) use; 148 (B200) when no device can be queried.
 */
int streamkl_num_sms(void);

/*
 * y[i] = 2^x[i] for i < n by one of the two exponential paths the kernels use, for checking
 * their accuracy; no part of the KL computation.  kind 0: ex2.approx on the exponential unit
 * (subnormal results flushed to zero); kind 1: the FMA-pipe polynomial (x clamped at -126,
 * worst relative error of the fit 2.7e-6 for -126 <= x <= 0; meant for x <= 0).
 *   x, y : device arrays of n fp32 (caller-owned; y may not overlap x).
 * One kernel on `stream`.  Returns STREAMKL_ERR_INVALID_ARG for a bad kind, n < 0 or a NULL
 * array with n > 0; n = 0 launches nothing.
 */
int streamkl_eval_exp2(int kind, const float* x, float* y, long long n, void* stream);

/*
 * Effective SM clock probe; no part of the KL computation.  Under the board's power cap
 * the SM clock runs below its maximum while heavy kernels run, so a kernel's time depends
 * on that clock; this records it while other work runs.  Launches one 32-thread CTA on
 * `stream` (meant for a stream of its own, concurrent with the work being timed: it needs
 * no shared memory and sleeps between samples, so it fits beside every kernel of this
 * library on one SM) whose first thread writes, every `interval_ns`, the pair
 * (%globaltimer in ns, clock64 of its SM) until `duration_ns` has passed or `max_pairs`
 * pairs are written.  The effective clock between two pairs is
 * delta(clock64) / delta(ns) in GHz.
 *   samples  : device buffer of 2 + 2 * max_pairs int64, 8-byte aligned; on completion
 *              samples[0] = pairs written, samples[1] = 0, pair i at samples[2 + 2i],
 *              samples[3 + 2i].
 *   duration : 1 us to 10 s; interval: 1 us to duration; max_pairs >= 2.
 * Returns STREAMKL_ERR_INVALID_ARG for an argument outside these ranges (nothing launched),
 * STREAMKL_ERR_UNSUPPORTED for a misaligned buffer.
 */
int streamkl_probe_clock(long long duration_ns, long long interval_ns, long long* samples,
                         int max_pairs, void* stream);

/* Static text for a status code (never NULL). */
const char* streamkl_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the device status word of the current
 * device.  Returns STREAMKL_OK, STREAMKL_ERR_TIMEOUT (a kernel abandoned a pipeline wait
 * and left its outputs undefined) or STREAMKL_ERR_CUDA (the synchronisation itself failed;
 * cudaGetLastError text is available through streamkl_last_cuda_error).
 */
int streamkl_device_status(void* stream);

/*
 * Self-test of the bounded waits that guard every pipeline kernel (no part of the KL
 * computation).  Runs one small kernel on `stream` and waits for it: two threads wait on
 * two mbarriers, the second starting 0.5 s after the first.
 *   starve == 0: the barriers are completed before anyone waits; returns STREAMKL_OK.
 *   starve != 0: nothing completes them.  The first wait gives up after the library's
 *     wait limit (2 s), records STREAMKL_ERR_TIMEOUT and raises the CTA's abort flag; the
 *     second wait sees the flag and gives up at once.  Returns STREAMKL_ERR_TIMEOUT.
 * Nothing faults or traps; the context stays usable.  The device status word is read and
 * cleared like streamkl_device_status does.  If waited_ns is not NULL it receives the
 * nanoseconds each of the two waits took.  Returns STREAMKL_ERR_CUDA if a CUDA call
 * failed.  Blocks the calling host thread for up to about 2.5 s.
 */
int streamkl_selftest_watchdog(int starve, long long* waited_ns, void* stream);

/* Text of the last CUDA error the library saw on this host thread ("" if none). */
const char* streamkl_last_cuda_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int streamkl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STREAMKL_H */
