/*
 * bsfa.h - C ABI of the B200 (sm_100a) Block Sparse Flash Attention prefill forward.
 *
 * The operation ("Block Sparse Flash Attention", §4 Method, §4.1 Gating
 * Mechanism, §4.4 Algorithm and Implementation, App. B.2): tiled online-softmax
 * attention that computes every score S = Q K^T / sqrt(d) exactly. For each
 * (query tile i, key block j) it takes the block maximum s_max(i,j) over the
 * valid entries; when s_max(i,j) < tau[h] the block's values are not loaded, the
 * PV product is not run and the running statistics (m, l, O) are not updated.
 * Diagonal blocks bypass the gate. The result is therefore the softmax over each
 * query tile's kept key set.
 *
 * Definitions used by every entry point:
 *   - Query tile i holds rows [i*Bq, min((i+1)*Bq, N)); key block j holds keys
 *     [j*Bk, min((j+1)*Bk, N)). There are M_Q = ceil(N/Bq) tiles and
 *     M_KV = ceil(N/Bk) blocks (App. B.2); N need not be a multiple of either.
 *   - Causal: key c is valid for query r when c <= r. A block is visible when some
 *     entry is valid; it is diagonal (gate bypassed) when it is visible and also
 *     holds an invalid entry. Non-causal ("bidirectional", App. B.3): the diagonal
 *     blocks are those whose key range overlaps the tile's query range.
 *   - tau is in units of the scaled score q.k/sqrt(d); a block whose maximum
 *     equals tau is kept. tau = -INFINITY gives dense attention.
 *   - GQA: query head h reads KV head h / (Hq / Hkv).
 *
 * Thread safety: entry points may be called from several host threads; calls on
 * the same stream are ordered by the stream. The library allocates nothing per
 * call; it keeps one device status word per device (and, for bsfa_forward_host,
 * two copy streams, a second compute stream and their events per device,
 * created on first use).
 *
 * The status word is shared by every kernel the library runs on a device,
 * whatever stream or host thread launched it: bsfa_get_status reports (and
 * clears) a bounded-wait failure of ANY of them, not only of the caller's own
 * stream. Callers that run forwards on several streams of one device and need
 * to tell their failures apart must serialise their bsfa_get_status calls with
 * their launches. Concurrent bsfa_forward_host calls on one device are
 * serialised inside the library (each holds the device's copy pipeline from its
 * first copy to its last).
 */
#ifndef BSFA_H_
#define BSFA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSFA_OK = 0,
  BSFA_ERR_INVALID_ARG = 1,     /* null pointer, non-positive size, Hq % Hkv != 0, misaligned pointer */
  BSFA_ERR_UNSUPPORTED = 2,     /* D, Bq, Bk or N outside the supported set, or no sm_100 device */
  BSFA_ERR_CUDA = 3,            /* a CUDA runtime or driver call failed (see bsfa_last_error) */
  BSFA_ERR_DEVICE_TIMEOUT = 4   /* a kernel gave up on a bounded wait (reported by bsfa_get_status) */
} bsfa_status;

/*
 * bsfa_forward - BSFA prefill forward for a batch of heads, asynchronous on `stream`.
 *
 *   q          bf16 [B, N, Hq,  D], contiguous, device memory, 16-byte aligned (read)
 *   k          bf16 [B, N, Hkv, D], contiguous, device memory, 16-byte aligned (read)
 *   v          bf16 [B, N, Hkv, D], contiguous, device memory, 16-byte aligned (read; only
 *              the blocks some query tile keeps are loaded)
 *   tau        fp32 [Hq], device memory: one threshold per query head (§4.1; the paper's
 *              table indexed by layer, head and position is reduced to one value per head)
 *   out        bf16 [B, N, Hq, D], contiguous, device memory, 16-byte aligned (written)
 *   lse        fp32 [B, Hq, N], device memory, natural-log logsumexp over each row's kept
 *              set (written); NULL skips it
 *   block_mask uint8 [B, Hq, M_Q, M_KV], device memory (written); NULL turns the debug
 *              output off. Codes: 0 skipped by the gate, 1 kept by the gate, 2 diagonal
 *              (forced keep), 3 not visible. The library fills it with 3 first.
 *   B, Hq, Hkv, N, D   sizes; Hq % Hkv == 0
 *   Bq, Bk     query-tile and key-block sizes (the paper's B_M and B_N)
 *   causal     nonzero for causal prefill, zero for bidirectional attention
 *   stream     a cudaStream_t (NULL = the legacy default stream)
 *
 * Supported: D in {64, 128}; Bq, Bk in {64, 128}; any N >= 1 with at most 4096
 * key blocks (M_KV <= 4096); an sm_100 device. Rows and keys past N inside the
 * last tile or block are padding: they never enter a block maximum or a softmax,
 * and no output row past N is written. The caller owns every buffer; results are valid once the
 * stream has reached the call. Returns BSFA_OK once the kernel is enqueued;
 * argument errors are returned before any CUDA call is made. A kernel that gives
 * up on a bounded internal wait leaves `out` undefined and sets the device
 * status word that bsfa_get_status reports.
 */
bsfa_status bsfa_forward(const void* q, const void* k, const void* v, const float* tau, void* out, float* lse,
                         uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal,
                         void* stream);

/*
 * bsfa_forward_tau_table - bsfa_forward with one threshold per (query head,
 * query tile): the per-position thresholds of §4.1 / §4.2 ("thresholds
 * calibrated per (layer, head, position)").
 *
 *   tau_table  fp32 [Hq, tau_tiles], device memory, row-major (read). Query tile i
 *              of head h is gated against tau_table[h * tau_tiles + min(i, tau_tiles - 1)]:
 *              a sequence longer than the calibrated length reuses the last
 *              calibrated position (App. B.3 "Practical considerations"). One layer
 *              and sparsity level of the paper's table T[S, L, H, ceil(N_max/B_M)] is
 *              the contiguous slice T[level, layer], with tau_tiles = ceil(N_max/B_M);
 *              the table must be calibrated with the same Bq.
 *   tau_tiles  number of calibrated query tiles per head, >= 1
 *
 * Every other argument, the supported set and the error behaviour are those of
 * bsfa_forward; tau_tiles <= 0 returns BSFA_ERR_INVALID_ARG.
 */
bsfa_status bsfa_forward_tau_table(const void* q, const void* k, const void* v, const float* tau_table, int tau_tiles,
                                   void* out, float* lse, uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D,
                                   int Bq, int Bk, int causal, void* stream);

/*
 * bsfa_forward_gap - the same forward with a different gate, for comparison: the
 * gap to the running maximum that the paper sets against its own threshold
 * (§3 Related Work, on BLASST and SpargeAttention). The query tile visits its
 * visible key blocks in order; each row r keeps M_r, the maximum of its scaled
 * scores over the blocks kept so far (-inf before the first). A block that does
 * not bypass the gate is kept when some row with a valid entry in it has a block
 * maximum >= M_r - gamma[h]; kept blocks (diagonal ones included) then raise M_r.
 * gamma may have either sign: a negative gamma keeps only blocks that raise
 * some row's maximum by at least -gamma.
 *
 *   gamma      fp32 [Hq], device memory, in scaled-score units (q.k / sqrt(d))
 *
 * Every other argument, the supported set and the error behaviour are those of
 * bsfa_forward; block_mask codes 0 and 1 record this gate's decisions.
 */
bsfa_status bsfa_forward_gap(const void* q, const void* k, const void* v, const float* gamma, void* out, float* lse,
                             uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal,
                             void* stream);

/*
 * bsfa_forward_heads - bsfa_forward for the query heads of KV heads
 * [kv_begin, kv_begin + kv_count) only: one head shard of the layer, for
 * splitting a layer's KV groups across GPUs. Heads are independent problems,
 * so the shards need no exchange. All tensors keep their full [.., Hq or Hkv, ..]
 * shapes and strides; only the selected heads' rows of out and lse are written.
 * The block mask, if given, is filled with 3 whole, then written for the
 * selected heads. 0 <= kv_begin, 1 <= kv_count, kv_begin + kv_count <= Hkv,
 * else BSFA_ERR_INVALID_ARG; everything else as bsfa_forward.
 */
bsfa_status bsfa_forward_heads(const void* q, const void* k, const void* v, const float* tau, void* out, float* lse,
                               uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal,
                               int kv_begin, int kv_count, void* stream);

/*
 * bsfa_forward_rows - bsfa_forward for query rows [row_begin, row_end) of every
 * batch entry and head only. Every (query tile, key block) pair of those rows is
 * computed exactly as the whole-layer call computes it ("Block Sparse Flash
 * Attention" §4.4: query tiles are independent), so a layer can be computed in
 * row chunks, e.g. while later rows are still being copied in. A chunk reads the
 * K/V rows it attends to: [0, row_end) with the causal mask, all N without it.
 * All tensors keep their full shapes and strides; only the selected rows of out
 * and lse are written. The block mask, if given, is filled with 3 whole, then
 * written for the selected query tiles.
 *
 *   row_begin   a multiple of 256, >= 0
 *   row_end     row_begin < row_end <= N
 *
 * Else BSFA_ERR_INVALID_ARG; everything else as bsfa_forward.
 */
bsfa_status bsfa_forward_rows(const void* q, const void* k, const void* v, const float* tau, void* out, float* lse,
                              uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal,
                              int row_begin, int row_end, void* stream);

/*
 * bsfa_forward_host - bsfa_forward on HOST buffers, with the copies overlapped
 * with the kernel. K and V go up first, whole (one copy each). The query rows
 * follow in `chunks` runs of whole 256-row units, the same rows of every batch
 * entry, one copy per run; the runs shrink towards the end (cumulative share
 * 1 - (1 - c/chunks)^2 after run c, at least one unit each), so little is left
 * after the last upload. The kernel computes a run's rows (bsfa_forward_rows) as
 * soon as they have landed, alternating between the caller's stream and a second
 * compute stream, and the run's out rows come back on a second copy stream while
 * the next run computes; lse (head-major, so a run's rows would be B * Hq short
 * pieces) comes back whole after the last run. Asynchronous: everything is done
 * once `stream` reaches the call.
 *
 *   q_host, k_host, v_host, tau_host   inputs in host memory, the layouts of
 *                                      bsfa_forward; page-locked (pinned) memory is
 *                                      needed for the copies to overlap
 *   out_host, lse_host                 results in host memory (lse_host may be NULL)
 *   q_dev ... lse_dev                  device buffers of bsfa_forward's shapes, owned
 *                                      by the caller (lse_dev NULL iff lse_host is)
 *   chunks                             1 <= chunks <= min(ceil(N / 256), 64)
 *
 * The library creates two copy streams, a second compute stream and their
 * events once per device and reuses them; calls on one device share them: a call holds them (a host lock)
 * while it enqueues, so concurrent calls from several host threads are
 * serialised and never consume each other's events.
 * Errors as bsfa_forward; BSFA_ERR_INVALID_ARG for a bad chunk count or a
 * missing buffer.
 */
bsfa_status bsfa_forward_host(const void* q_host, const void* k_host, const void* v_host, const float* tau_host,
                              void* out_host, float* lse_host, void* q_dev, void* k_dev, void* v_dev, float* tau_dev,
                              void* out_dev, float* lse_dev, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk,
                              int causal, int chunks, void* stream);

/*
 * bsfa_forward_varlen - bsfa_forward over a packed batch of sequences of
 * different lengths (mixed-length prefill). Sequence e holds rows
 * [cu_seqlens[e], cu_seqlens[e+1]) of the packed tensors; each sequence is its
 * own attention problem, tiled from its own first row (App. B.2 tiling applied
 * per sequence).
 *
 *   q          bf16 [total, Hq,  D], contiguous, device memory, 16-byte aligned (read)
 *   k, v       bf16 [total, Hkv, D], contiguous, device memory, 16-byte aligned (read)
 *   cu_seqlens int32 [nseq + 1], device memory: cu_seqlens[0] = 0, non-decreasing,
 *              cu_seqlens[nseq] <= total. Offsets outside [0, total] are clamped and a
 *              sequence longer than max_seqlen is cut to max_seqlen (its rows past that
 *              are not written), so bad offsets cannot make the kernel leave the buffers.
 *   nseq       number of sequences, >= 1
 *   max_seqlen length of the longest sequence (it sizes the grid), >= 1, with
 *              ceil(max_seqlen / Bk) <= 4096
 *   tau        fp32 [Hq], device memory (one threshold per head)
 *   out        bf16 [total, Hq, D], device memory (written for the rows of every sequence)
 *   lse        fp32 [Hq, total], device memory, or NULL
 *   block_mask uint8 [nseq, Hq, ceil(max_seqlen/Bq), ceil(max_seqlen/Bk)], device
 *              memory, or NULL; entries past a sequence's own tiles stay 3
 *   total      total rows of the packed tensors
 *
 * Hq, Hkv, D, Bq, Bk, causal and stream, the supported set and the error
 * behaviour are those of bsfa_forward.
 */
bsfa_status bsfa_forward_varlen(const void* q, const void* k, const void* v, const int* cu_seqlens, int nseq,
                                int max_seqlen, const float* tau, void* out, float* lse, uint8_t* block_mask,
                                int total, int Hq, int Hkv, int D, int Bq, int Bk, int causal, void* stream);

/*
 * bsfa_validate - the shape checks of bsfa_forward, host only (no CUDA call).
 * Returns BSFA_OK, BSFA_ERR_INVALID_ARG or BSFA_ERR_UNSUPPORTED.
 */
bsfa_status bsfa_validate(int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal);

/*
 * bsfa_get_status - synchronise `stream`, then read and clear the device status
 * word of the current device. Returns BSFA_ERR_DEVICE_TIMEOUT when a kernel gave
 * up on a bounded wait since the last call, BSFA_ERR_CUDA when the
 * synchronisation itself failed, else BSFA_OK. The word is one per device: a
 * failure of a kernel launched on another stream of the same device is reported
 * here too (and cleared), even if that stream has not finished.
 */
bsfa_status bsfa_get_status(void* stream);

/*
 * bsfa_get_debug_counts - synchronise `stream`, then read and clear the debug
 * counters of the current device: the V tiles loaded and the PV products issued
 * by every launch that wrote a block mask (block_mask != NULL) since the last
 * call. Launches without a block mask count nothing and carry no counting code.
 * They show the skip of §4.3 / §4.4 directly: a CTA loads the V tile of block j
 * once if some of its query tiles kept j, and issues one PV product per (128-row
 * slot, kept block). Like the status word, the counters are one pair per device,
 * shared by all streams and host threads.
 *
 *   v_tiles, pv_products   host pointers, written (must be non-null)
 *
 * Returns BSFA_ERR_INVALID_ARG for a null pointer, BSFA_ERR_CUDA if the
 * synchronisation or a copy fails, else BSFA_OK.
 */
bsfa_status bsfa_get_debug_counts(void* stream, unsigned long long* v_tiles, unsigned long long* pv_products);

/*
 * bsfa_selftest_lost_arrival - exercise the failure path on the device: one
 * thread waits, through the forward kernel's bounded wait, on a barrier that
 * nothing arrives on (the shape of a lost arrival). After the wait's time limit
 * (about 2 s) the kernel sets the device status word and exits normally; no
 * trap, the context stays usable. Asynchronous on `stream`; the next
 * bsfa_get_status(stream) returns BSFA_ERR_DEVICE_TIMEOUT.
 */
bsfa_status bsfa_selftest_lost_arrival(void* stream);

/* bsfa_status_string - a static, human-readable name for a status code. */
const char* bsfa_status_string(bsfa_status s);

/*
 * bsfa_last_error - details of the last failure on the calling host thread
 * (a static thread-local buffer, valid until the thread's next call).
 */
const char* bsfa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BSFA_H_ */
