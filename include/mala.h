/*
 * mala.h -- C ABI of the MALA (MassAlloc Attention) library for NVIDIA B200
 * (sm_100a).
 *
 * MALA is causal softmax attention that computes every legal QK tile but
 * skips the post-score work of a tile when, for every valid query row of the
 * tile, the tile's largest per-key contribution ratio is below tau / Lq
 * (Lq = number of keys the query can see). Sources: the pages on arXiv
 * 2609.32712 "MassAlloc Attention: Let Attention Allocate Its Own Compute" --
 * agihunt.info summary (rule, forward and backward paragraphs) and the
 * jaehun.me review, sections "One tolerance governs everything", "Forward:
 * online sparse softmax" and "Backward: offline sparse probabilities".
 *
 * Conventions shared by every call
 *  - Layout: Q, K, V, O, dO, dQ, dK, dV are [B][H][L][d] contiguous, d
 *    innermost; LSE is [B][H][L] float32. The decode cache is
 *    [B][Hkv][Lc][d]; the decode query and output are [B][Hq][d]. Query head
 *    h uses KV head h / (Hq / Hkv).
 *  - All data pointers are DEVICE pointers, 16-byte aligned. The caller owns
 *    every buffer (inputs, outputs, workspace); the library allocates no
 *    device memory and keeps no state between calls except one device-side
 *    status word per GPU (see mala_check).
 *  - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous on that stream; none synchronizes.
 *  - scale <= 0 selects 1/sqrt(d). tau >= 0 and finite; tau = 0 never skips
 *    (exact FullAttn, the pages' tau -> 0 limit). tau < 0 or NaN is
 *    MALA_ERR_INVALID_ARG.
 *  - Argument errors are detected on the host and returned before anything
 *    is launched. A failed launch returns MALA_ERR_CUDA. A device-side wait
 *    that exceeds its time limit (about two seconds) records a status that
 *    mala_check reports as MALA_ERR_TIMEOUT; kernels never trap.
 *  - Optional trace outputs (pass NULL to skip them; device pointers):
 *      kept_tiles: int32 counts of kept tiles (layout per call below);
 *      keep_bits:  uint32 bitmask, bit (j % 32) of word [.., row, j / 32]
 *                  set iff tile (row, j) was kept. Both are written in full
 *                  by the call (no pre-zeroing needed).
 */
#ifndef MALA_H
#define MALA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MALA_OK = 0,
  MALA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned, tau < 0 */
  MALA_ERR_UNSUPPORTED = 2, /* (dtype, d, tile) combination not built */
  MALA_ERR_CUDA = 3,        /* CUDA runtime error at launch or check */
  MALA_ERR_TIMEOUT = 4,     /* a device-side wait ran out (see mala_check) */
  MALA_ERR_TOO_LARGE = 5    /* shape needs more than the built-in scratch */
} mala_status;

typedef enum { MALA_F32 = 0, MALA_BF16 = 1 } mala_dtype;

/*
 * Forward pass (training forward / prefill).
 *
 * Per (b, h, query block i of `tile` rows) the key tiles j = i, i-1, ..., 0
 * are visited from the diagonal toward earlier keys. Every legal tile's
 * scores S = scale * Q_i K_j^T are computed. With the running row max m, the
 * retained mass l (online softmax over the tiles kept so far) and the tile's
 * row max mt, the tile is skipped iff every valid row r satisfies
 *     mt_r - m_r - ln l_r  <  ln tau - ln (r + 1)
 * (the log form of exp(mt - m) / l < tau / Lq; equality keeps). A skipped
 * tile leaves m, l and O untouched and its V is never read; a kept tile does
 * the standard online-softmax update. The diagonal tile is always kept.
 * Sources: agihunt.info summary, forward paragraph; jaehun.me review,
 * "Forward: online sparse softmax".
 *
 * Inputs  Q: [B][H][L][d], K, V: [B][Hkv][L][d] of dtype dt. Grouped
 *         query heads: query head h reads key/value head h / (H / Hkv);
 *         Hkv = H is ordinary multi-head attention. Every query head applies
 *         the rule to its own rows.
 * Outputs O: [B][H][L][d] of dtype dt, softmax over the retained tiles;
 *         LSE: [B][H][L] float32, natural-log normalizer m + ln l over the
 *         retained keys (with O, the only state backward needs);
 *         O_f32 (may be NULL): [B][H][L][d] float32, the same output before
 *         rounding to dt. Pass it to mala_bwd: the backward's row terms
 *         D = <dO, O> feed dQ through a sum over keys whose rows cancel, so
 *         D computed from a bf16-rounded O costs dQ percents of accuracy when
 *         keys share a large common component.
 * Trace   kept_tiles: [B][H][nb] kept key tiles per query block;
 *         keep_bits: [B][H][nb][ceil(nb/32)], row = query block, bit = key
 *         block. nb = ceil(L / tile).
 * Supported: (dt, d, tile) in {(MALA_BF16, 128, 128), (MALA_F32, 32|64|128, 64)};
 *            any L >= 0 (a ragged last block is masked), B, H >= 1, H % Hkv
 *            == 0 (Hkv < H: MALA_BF16 only).
 * Memory: nothing but O, LSE (and O_f32 when given) is written; no score,
 *         row maximum or selection mask outlives the call.
 */
mala_status mala_fwd(const void* Q, const void* K, const void* V, void* O,
                     float* LSE, float* O_f32, int B, int H, int Hkv, int L,
                     int d, mala_dtype dt, float tau, int tile, float scale,
                     int32_t* kept_tiles, uint32_t* keep_bits, void* stream);

/*
 * Prefill of chunks appended to KV caches, several sequences packed (prefill
 * and decode use the same tau: agihunt.info summary, "one tau for prefill and
 * decode").
 *
 * Sequence b's new queries are tokens [cu_seqlens_q[b], cu_seqlens_q[b+1])
 * of Q; its keys and values, cached ones first, are tokens
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]) of K and V, with Lk_b >= Lq_b. Query
 * r of the chunk sits at position off_b + r (off_b = Lk_b - Lq_b), sees keys
 * 0 .. off_b + r and has Lq = off_b + r + 1 in the threshold. Query blocks
 * are the chunk's own 128-row blocks; key tiles are aligned to them (tile k
 * starts at position off_b + 128 (k - koff_b), koff_b = ceil(off_b / 128),
 * positions below 0 do not exist), so a chunk whose cache is a whole number
 * of tiles reproduces the full prefill's rows exactly. Each block visits its
 * diagonal tile (always kept) and then the earlier tiles, with the rule of
 * mala_fwd.
 *
 * Inputs  Q: [total_q][H][d] bf16; K, V: [total_k][Hkv][d] bf16 (query head
 *         h reads key/value head h / (H / Hkv)); cu_seqlens_q,
 *         cu_seqlens_k: device int32 [batch + 1], non-decreasing from 0.
 *         max_seqlen_q >= every Lq_b (blocks past it are not computed),
 *         max_seqlen_k >= every Lk_b (trace layout). A sequence with
 *         Lk_b < Lq_b is left untouched.
 * Outputs O: [total_q][H][d] bf16; LSE: [H][total_q] float32.
 * Trace   kept_tiles: [batch][H][nbq] with nbq = ceil(max_seqlen_q / 128);
 *         keep_bits: [batch][H][nbq][mala_varlen_trace_words(...)], bit k of
 *         a row = key tile k kept.
 * Supported: d = 128, tile = 128, H % Hkv == 0, batch * H <= 65535.
 */
mala_status mala_fwd_varlen(const void* Q, const void* K, const void* V, void* O,
                            float* LSE, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, int batch,
                            int max_seqlen_q, int max_seqlen_k, int total_q,
                            int total_k, int H, int Hkv, int d, float tau,
                            int tile, float scale, int32_t* kept_tiles,
                            uint32_t* keep_bits, void* stream);

/* 32-bit words per query block in mala_fwd_varlen's keep_bits. */
int mala_varlen_trace_words(int max_seqlen_q, int max_seqlen_k);

/* Bytes of device workspace mala_bwd needs: the row terms D (float32
 * [B][H][L]), the float32 dQ accumulator [B][H][L][d] and the per-tile keep
 * bits of the backward's test pass (B*H*nb*ceil(nb/32) words for nb =
 * ceil(L/64)), each rounded up to 256 bytes, and 256 bytes for the work
 * pass's column counter. */
size_t mala_bwd_workspace_bytes(int B, int H, int L, int d);

/*
 * Backward pass.
 *
 * Uses the forward's final LSE instead of replaying its partial normalizers.
 * Every legal tile's scores are recomputed, and tile (i, j) is skipped iff
 * every valid row r satisfies
 *     max_c S_rc - LSE_r  <  ln tau - ln (r + 1).
 * Only O and LSE (or O_f32) come from the forward: no mask, score or row
 * maximum is carried between the passes, and there is no forced keep. In
 * exact arithmetic the kept set is inside the forward's. Kept tiles do the standard work with
 * P = exp(S - LSE), D_r = <dO_r, O_r>: dV_j += P^T dO_i, dP = dO_i V_j^T,
 * dS = P o (dP - D), dQ_i += scale dS K_j, dK_j += scale dS^T Q_i.
 * Sources: agihunt.info summary, backward paragraph; jaehun.me review,
 * "Backward: offline sparse probabilities".
 *
 * Inputs  Q, O, dO: [B][H][L][d], K, V: [B][Hkv][L][d] of dtype dt (grouped
 *         heads as in mala_fwd); LSE from mala_fwd;
 *         O_f32 (may be NULL): the float32 output of mala_fwd, used for the
 *         row terms D instead of O when given.
 * Outputs dQ: [B][H][L][d]; dK, dV: [B][Hkv][L][d], summed over the query
 *         heads of each group; dtype dt (fully overwritten).
 * workspace: device buffer of at least mala_bwd_workspace_bytes(B,H,L,d)
 *         bytes, 256-byte aligned, contents ignored on entry.
 * Trace   kept_tiles: [B][H][nb] kept query blocks per key block;
 *         keep_bits: [B][H][nb][ceil(nb/32)], row = query block i, bit = key
 *         block j.
 * Supported: as mala_fwd.
 */
mala_status mala_bwd(const void* Q, const void* K, const void* V,
                     const void* O, const float* O_f32, const void* dO,
                     const float* LSE, void* dQ, void* dK, void* dV,
                     void* workspace,
                     size_t workspace_bytes, int B, int H, int Hkv, int L, int d,
                     mala_dtype dt, float tau, int tile, float scale,
                     int32_t* kept_tiles, uint32_t* keep_bits, void* stream);

/* Bytes of device workspace mala_decode needs (per-tile statistics, the
 * kept-tile lists, the final normalizers and a float32 output accumulator),
 * each part rounded up to 256 bytes. */
size_t mala_decode_workspace_bytes(int B, int Hq, int Hkv, int Lc, int d);

/*
 * One decode step with the same rule (agihunt.info summary: one tau for
 * prefill and decode; the KV cache is kept whole).
 *
 * The cache holds Lc keys per (b, kv head) including the current token, so
 * Lq = Lc. Key tiles of 128 positions are aligned from position 0 and
 * visited newest first; the newest tile is always kept. With per_head = 0
 * the rows of a tile are the G = Hq / Hkv query heads that share the KV
 * head, and the tile is skipped iff every one of them is below the threshold
 * (tile granularity is conservative). With per_head = 1 every query head
 * applies the test alone, with its own running statistics (finer skipping;
 * a tile's K and V are still read once for all heads that kept it). Kept
 * tiles update the per-head online softmax; the output is softmax over the
 * kept tiles.
 *
 * Inputs  q: [B][Hq][d] bf16; Kcache, Vcache: [B][Hkv][Lc][d] bf16.
 * Output  o: [B][Hq][d] bf16.
 * workspace: at least mala_decode_workspace_bytes(B,Hq,Hkv,Lc,d) bytes.
 * Trace   kept_tiles: [B][Hkv]; keep_bits: [B][Hkv][ceil(nt/32)], nt =
 *         ceil(Lc / 128); with per_head = 1, [B][Hq] and [B][Hq][ceil(nt/32)].
 * Supported: d = 128, Hq % Hkv == 0, 1 <= Hq / Hkv <= 8, B * Hkv <= 4095,
 *            Lc >= 1.
 */
mala_status mala_decode(const void* q, const void* Kcache, const void* Vcache,
                        void* o, int B, int Hq, int Hkv, int Lc, int d,
                        float tau, float scale, int per_head, void* workspace,
                        size_t workspace_bytes, int32_t* kept_tiles,
                        uint32_t* keep_bits, void* stream);

/* Size of the device scratch array that mala_decode_noalloc uses in place
 * of a caller's workspace (8 MiB; B = 16, Hq = 32, Hkv = 8, Lc = 131072 needs
 * about 4.8 MiB). */
#define MALA_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * mala_decode without a workspace argument, for callers that cannot allocate
 * device memory. The paper has no counterpart: this is an interface choice.
 *
 * Who needs it: code whose host program hands it only the buffers it reads
 * and writes and keeps every other byte of device memory for itself (a plugin
 * or custom operator inside an inference server with its own memory pool, a
 * runtime that reserves the GPU's memory at start-up). There a cudaMalloc
 * either fails or forces the pool to give memory back, and a serving loop
 * cannot afford that in the middle of a step.
 *
 * Scratch: a file-scope __device__ array of MALA_DECODE_NOALLOC_SCRATCH_BYTES
 * bytes inside this library. Every GPU that loads the library holds it until
 * the process exits. The first call on a device, with that device current,
 * looks up the array's device address (cudaGetSymbolAddress) and caches it
 * with the unique ID of the current context; a call in another context of
 * that device (after cudaDeviceReset, say) looks it up again. Make the first
 * call in a context before any stream capture begins. The call itself
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * routine.
 *
 * All calls on a device share the one array and it keeps the last call's
 * contents; the kernels clear the part that must start at zero (the float32
 * output accumulator) in every call. Calls that overlap on the GPU (two
 * streams, or two host threads, at once) race on the array: serialise them.
 *
 * Arguments, layouts, outputs and the rule are those of mala_decode.
 * Errors: as mala_decode, and MALA_ERR_TOO_LARGE, before any launch, when
 * mala_decode_workspace_bytes(B, Hq, Hkv, Lc, d) exceeds
 * MALA_DECODE_NOALLOC_SCRATCH_BYTES. MALA_ERR_CUDA if the array's address
 * cannot be found on the current device.
 */
mala_status mala_decode_noalloc(const void* q, const void* Kcache,
                                const void* Vcache, void* o, int B, int Hq,
                                int Hkv, int Lc, int d, float tau, float scale,
                                int32_t* kept_tiles, uint32_t* keep_bits,
                                void* stream);

/*
 * Synchronizes `stream`, then reads and clears this GPU's device status word.
 * Returns MALA_ERR_CUDA if the stream reported an error (or a kernel found
 * its shared memory laid out unusably and did nothing), MALA_ERR_TIMEOUT if a
 * kernel gave up on a wait since the last check, MALA_OK otherwise.
 */
mala_status mala_check(void* stream);

/*
 * Diagnostic of the timeout path (no counterpart in the pages): launches one
 * thread on `stream` that waits, with the bounded wait every kernel uses
 * (about two seconds of %globaltimer), on a barrier that nothing arrives on.
 * The wait runs out and records a timeout in the device status word, so the
 * next mala_check returns MALA_ERR_TIMEOUT and clears it. Nothing traps, no
 * memory is touched but the status word, and the context stays usable.
 * Returns MALA_ERR_CUDA if the launch fails, MALA_OK otherwise.
 */
mala_status mala_selftest_wait(void* stream);

/* Static, human-readable name of a status code. */
const char* mala_status_string(mala_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
int mala_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MALA_H */
