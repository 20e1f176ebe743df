/*
 * spec_verify.h -- C ABI of libspecverify: batched lossless speculative-
 * sampling verification, two-stage (L_d -> L_i -> L_f) verification over a
 * window, and the paged-KV commit that follows it, on NVIDIA B200 (sm_100a).
 *
 * Where the operations come from
 *   [HS]  "HiSpec: Hierarchical Speculative Decoding for LLMs", gist.science
 *         summary of arXiv 2510.01336: section 2 "Methodik" -- Kernmechanismus
 *         (the exits L_d, L_i ~ 1/4 depth, L_f) and the bullets "Verlustfreie
 *         Garantie" (two-stage lossless check), "Dynamische
 *         Verifizierungsrichtlinie" (window of N_i = 4), "Wiederverwendung von
 *         KV-Cache und versteckten Zustaenden" (buffer, then drop rejected
 *         entries) and "Unterstuetzung fuer Batch-Inferenz" (paged attention,
 *         block tables, per-sequence acceptance without padding).
 *   [SSD] "Speculative Speculative Decoding", gist.science summary of arXiv
 *         2603.03251, Technische Zusammenfassung section 2 item 1 (an outcome
 *         is the accepted count plus a bonus token) and section 3.B (residual
 *         distribution proportional to the target-minus-draft difference).
 *   [SV]  "Optimierung der Inferenzgeschwindigkeit von Sprachmodellen durch
 *         spekulative Dekodierung" (mind-verse.de), SVIP paragraphs: the
 *         entropy of the draft-token distribution as the draft-length signal.
 * The pages print no formulas. The rules implemented are the standard
 * speculative-sampling rules they appeal to: with p = softmax(l_target / T)
 * and q = softmax(l_draft / T), draft x_j is accepted iff u_j * q_j(x_j) <
 * p_j(x_j); at the first rejection a the token is drawn from
 * normalize(max(0, p_a - q_a)) (from p_a if that mass is zero); if all K are
 * accepted a bonus token is drawn from p_K. A draw with weights w and uniform
 * u' takes the smallest v with sum_{t<=v} w_t > u' * sum_t w_t. T == 0 is the
 * greedy path: accept iff x_j == argmax l_target_j (ties: smallest id), emit
 * the argmax.
 *
 * Randomness: Philox4x32-10 (Salmon et al., SC'11), key = (seed & 0xffffffff,
 * seed >> 32), counter = (seq_id[b], round, position, stage); lane 0 is the
 * accept uniform, lane 1 the draw uniform; u = (2*(x >> 9) + 1) * 2^-24.
 * Stage 0 = draft step; stage 1 = chain verification and the first stage;
 * stage 2 = second stage.
 *
 * Conventions for every call
 *   - Pointers are DEVICE memory owned by the caller unless a comment says
 *     otherwise; the library allocates nothing and keeps no state between
 *     calls. Work is queued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream); no call synchronises the host.
 *   - Return value: SPEC_OK when the work was queued. Argument errors are
 *     found on the host before anything is launched (SPEC_EINVAL,
 *     SPEC_EWORKSPACE); a failed launch returns SPEC_ECUDA.
 *   - `dev_status` (device int32) records conditions only the device can see.
 *     It is sticky: kernels only ever store an error code into it, and only
 *     while it still holds SPEC_OK (first error wins). The caller sets it to
 *     SPEC_OK (0) and reads it when it wants. A commit does nothing while it
 *     holds an error.
 *   - Logit rows must start on 16-byte boundaries: the base pointers are
 *     16-byte aligned and the row stride times the element size is a
 *     multiple of 16 bytes. V itself may be any value >= 1.
 *   - Calls on different streams must use different workspaces; calls that
 *     share one workspace must not overlap on the GPU.
 */
#ifndef SPEC_VERIFY_H
#define SPEC_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPEC_OK = 0,
  SPEC_EINVAL = -1,      /* bad argument (host) / bad value (device, commit) */
  SPEC_ECUDA = -2,       /* a CUDA launch or API call failed                 */
  SPEC_EWORKSPACE = -3,  /* workspace missing, misaligned or too small       */
  SPEC_ENOBLOCKS = -4,   /* device: the free-block pool cannot cover a commit */
  SPEC_ETIMEOUT = -5,    /* device: a bounded wait ran out                   */
  SPEC_EDEVICE = -6      /* device: invalid input value in a verification
                            (draft id outside [0,V), temperature negative or
                            not finite, a row with no finite maximum, window
                            length out of range); the sequence's outputs are
                            set to -1 and the others are still computed      */
} spec_status;

typedef enum { SPEC_F32 = 0, SPEC_BF16 = 1 } spec_dtype;

/* Limits checked on the host. */
#define SPEC_MAX_K 256           /* drafts per sequence per call      */
#define SPEC_MAX_TOP 32          /* outcomes kept per sequence        */
#define SPEC_MAX_V (1 << 21)     /* vocabulary size                   */
#define SPEC_MAX_COMMIT_B 16384  /* sequences per paged commit        */
#define SPEC_MAX_FUSED_B 4096    /* sequences per fused verify+commit */
#define SPEC_MAX_CACHED 1024     /* cached tokens per sequence (Saguaro) */
#define SPEC_VP_MAX_RANKS 64     /* vocabulary shards (ranks)         */
#define SPEC_VP_ROW_BYTES 32     /* one row record of a shard         */
#define SPEC_VP_MASS_BYTES 16    /* one sequence's draw masses of a shard */

/* spec_verify_chain is one launch when V <= SPEC_SMALL_V (one CTA per
   sequence computes its rows' statistics itself, then checks and draws),
   two launches otherwise (row statistics over all SMs, then the check). */
#define SPEC_SMALL_V 4096

/* Bytes of workspace a call needs (aligned to 256 bytes). Ni == 0 sizes a
 * chain call, Ni > 0 a two-stage call. Returns 0 for invalid sizes. */
size_t spec_workspace_bytes(int B, int K, int V, int dtype, int Ni);

/* Static English text for a status code (host memory, never freed). */
const char* spec_status_string(int status);

/* ---------------------------------------------------------------------------
 * Chain verification ([HS] Kernmechanismus with one verifying exit; [SSD] 2.1)
 *
 * tgt   : target logits [B, K+1, V]; row (b, j) starts at element
 *         (b*(K+1) + j) * ld_tgt. Row j is the target law of slot j; row K
 *         gives the bonus token.
 * drf   : draft logits  [B, K, V];   row (b, j) starts at (b*K + j) * ld_drf.
 *         Not read for sequences with temperature 0.
 * dtype : SPEC_F32 or SPEC_BF16 (both tensors).
 * draft_tok   : int32 [B, K] drafted token ids.
 * temperature : float [B]: 0 (greedy) or within [1e-6, 1e6]; anything else
 *               marks the sequence invalid (SPEC_EDEVICE).
 * seed, seq_id (int32 [B]), round : Philox key and counter fields.
 * accept_len  : out int32 [B], a_b in [0, K] (-1 if the sequence is invalid).
 * out_tok     : out int32 [B, K+1]: drafts 0..a-1, then the drawn token at a,
 *               then -1.
 * diag        : optional out double [B, 4K+2] (NULL to skip): natural-log
 *               partition ln sum exp(l/T) of target rows 0..K, of draft rows
 *               0..K-1, p_j(x_j) for j < K, q_j(x_j) for j < K, and the mass
 *               Z of the final draw (sum max(0, p_a - q_a), or sum p_K for the
 *               bonus). NaN for greedy sequences.
 * ws, ws_bytes: workspace of at least spec_workspace_bytes(B, K, V, dtype, 0)
 *               bytes, 256-byte aligned. No initial contents are needed.
 * Equivalent to spec_chain_row_stats followed by spec_chain_decide. At
 * V <= SPEC_SMALL_V it runs as one launch that forms each row's statistics
 * in one pass per sequence instead (the sums are taken in another order, so
 * bits may differ from the two-launch form within the verification
 * tolerance); the workspace is checked but not written then.
 * ------------------------------------------------------------------------- */
int spec_verify_chain(const void* tgt, int64_t ld_tgt, const void* drf,
                      int64_t ld_drf, int dtype, int B, int K, int V,
                      const int32_t* draft_tok, const float* temperature,
                      uint64_t seed, const int32_t* seq_id, uint32_t round,
                      int32_t* accept_len, int32_t* out_tok, double* diag,
                      int32_t* dev_status, void* ws, size_t ws_bytes,
                      void* stream);

/* First half of spec_verify_chain: per-row softmax statistics (running max,
 * sum of exponentials, first argmax) over every target and draft row, split
 * over vocabulary tiles, written into the workspace. Same arguments. */
int spec_chain_row_stats(const void* tgt, int64_t ld_tgt, const void* drf,
                         int64_t ld_drf, int dtype, int B, int K, int V,
                         const float* temperature, int32_t* dev_status,
                         void* ws, size_t ws_bytes, void* stream);

/* Second half: combines the workspace statistics, runs the accept test on all
 * K positions, finds the first rejection and draws the resampled or bonus
 * token (re-reading only rows a of the target and draft). The logits,
 * temperatures and workspace must be those of the preceding
 * spec_chain_row_stats call. */
int spec_chain_decide(const void* tgt, int64_t ld_tgt, const void* drf,
                      int64_t ld_drf, int dtype, int B, int K, int V,
                      const int32_t* draft_tok, const float* temperature,
                      uint64_t seed, const int32_t* seq_id, uint32_t round,
                      int32_t* accept_len, int32_t* out_tok, double* diag,
                      int32_t* dev_status, void* ws, size_t ws_bytes,
                      void* stream);

/* ---------------------------------------------------------------------------
 * Two-stage verification, one round ([HS] Verlustfreie Garantie and
 * Dynamische Verifizierungsrichtlinie).
 *
 * lg_d, lg_i, lg_f : logits of the exits L_d, L_i, L_f, each [B, S, V] with
 *         S = Ni + K + 1; row (b, s) starts at element (b*S + s) * ld. Rows
 *         are indexed by slot since the last commit: slot s is the law of the
 *         s-th token after the committed prefix. The caller writes rows for
 *         slots >= win_len[b] before each call and leaves earlier slots
 *         unchanged within a window cycle.
 * Ni    : window size (>= 1). K: drafts per round (>= 1).
 * draft_tok : int32 [B, K], drafts for slots win_len[b] .. win_len[b]+K-1.
 * temperature, seed, seq_id, round : as for chain verification; stage one
 *         uses stage tag 1 and stage two stage tag 2, position = slot.
 * win_len : in/out int32 [B], tokens tentatively accepted in the current
 *         cycle (0 <= win_len < Ni on entry).
 * win_tok : in/out int32 [B, Ni+K], the window's tokens.
 * win_stat: in/out double [B, Ni+K, 2]: for each window slot, the largest raw
 *         logit m of its L_i row and ln sum_v exp((l_v - m)/T), buffered so
 *         stage two does not recompute them (the row's log-partition is
 *         m/T + the second value). NaN for greedy sequences.
 * Stage one checks the drafts against L_i (draft law L_d) at slots
 * w..w+K; its a1 accepted drafts and its drawn token join the window. If the
 * window then holds >= Ni tokens, stage two checks them against L_f (draft
 * law: L_i at each slot; bonus row: L_f at slot |W|), commits a2 + 1 tokens
 * and empties the window.
 * acc1    : out int32 [B] stage-one accepted count (-1 if invalid).
 * acc2    : out int32 [B] stage-two accepted count, -1 if stage two did not run.
 * commit_tok : out int32 [B, Ni+K+1] committed tokens then -1.
 * commit_n   : out int32 [B] number of committed tokens (0 if none).
 * diag    : optional out double [B, 4K + 3S + 1]: the chain layout for stage
 *         one, then ln-partition of L_f slots 0..S-1, p_f(tok_s) and
 *         q_i(tok_s) for s < S-1, and Z of stage two; NaN where not computed.
 * ws      : spec_workspace_bytes(B, K, V, dtype, Ni) bytes.
 * ------------------------------------------------------------------------- */
int spec_verify_hier(const void* lg_d, const void* lg_i, const void* lg_f,
                     int64_t ld, int dtype, int B, int K, int V, int Ni,
                     const int32_t* draft_tok, const float* temperature,
                     uint64_t seed, const int32_t* seq_id, uint32_t round,
                     int32_t* win_len, int32_t* win_tok, double* win_stat,
                     int32_t* acc1, int32_t* acc2, int32_t* commit_tok,
                     int32_t* commit_n, double* diag, int32_t* dev_status,
                     void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Paged-KV commit / rollback and pruning of buffered rows ([HS] KV-Cache
 * reuse and batch-inference bullets).
 *
 * block_tables : in/out int32 [B, max_blocks]; a sequence of length n owns
 *         entries 0 .. ceil(n / block_size) - 1.
 * seq_lens     : in/out int32 [B] current lengths.
 * base_len     : int32 [B] committed length before this round (<= seq_lens);
 *                NULL means base_len = seq_lens (grow only).
 * keep, keep_add : rows kept per sequence are keep[b] + keep_add (so a chain
 *         verification's accept_len with keep_add = 1 keeps a + 1 rows);
 *         must lie in [0, Kp1].
 * New length len' = base_len + kept. Entries no longer covered are freed
 * (sequences ascending, each table's tail in ascending index, pushed on
 * free_stack), then missing entries are allocated (sequences ascending,
 * popped from the top of the stack).
 * free_stack   : in/out int32 [num_blocks]; free_top: in/out device int32,
 *                number of valid entries (top of stack = free_stack[top-1]).
 * kv_stage : [B, Kp1, layers, 2, kv_heads, head_dim] 2-byte elements (the
 *            K and V rows staged for each verified token); kv_pool:
 *            [num_blocks, layers, 2, block_size, kv_heads, head_dim]. Kept row
 *            i of sequence b goes to position base_len[b] + i. Both NULL for a
 *            table-only commit. kv_heads*head_dim*2 must be a multiple of 16.
 * hid_stage: [B, Kp1, hidden] 2-byte elements; hid_out: [sum kept, hidden],
 *            sequences packed in order; hid_off: out int32 [B+1] exclusive
 *            scan of the kept counts (may be given without the hidden
 *            buffers). hidden*2 must be a multiple of 16. NULL to skip.
 * Every check (kept count, base_len, table entries and popped ids inside
 * [0, num_blocks), stack capacity, pool size) is made before anything is
 * changed; on failure *dev_status gets SPEC_EINVAL or SPEC_ENOBLOCKS and no
 * table, length, stack or buffer is modified.
 * ------------------------------------------------------------------------- */
int spec_commit_paged(int B, int block_size, int max_blocks,
                      int32_t* block_tables, int32_t* seq_lens,
                      const int32_t* base_len, const int32_t* keep,
                      int keep_add, int32_t* free_stack, int32_t* free_top,
                      int num_blocks, int Kp1, const void* kv_stage,
                      void* kv_pool, int layers, int kv_heads, int head_dim,
                      const void* hid_stage, void* hid_out, int32_t* hid_off,
                      int hidden, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Chain verification and the paged commit of its kept rows in one call
 * ([HS] Verlustfreie Garantie, KV-Cache reuse and batch-inference bullets).
 *
 * Same results as spec_verify_chain followed, on the same stream, by
 * spec_commit_paged with keep = accept_len, keep_add = 1 and Kp1 = K + 1
 * (a + 1 rows kept per sequence: the accepted drafts and the drawn token),
 * in three launches instead of four: the row statistics; one cluster per
 * sequence for the check and the draw, whose last sequence to finish its
 * accept test plans the commit from per-sequence records; the copy of the
 * kept K/V and hidden rows, which starts while the draws run, as soon as the
 * plan is written.
 * Arguments: those of spec_verify_chain (the logits, drafts, temperatures,
 * Philox key, accept_len, out_tok, diag, workspace) and of spec_commit_paged
 * (tables, lengths, base_len, stack, pool, stage and hidden buffers), with
 * the same layouts and ownership; B <= SPEC_MAX_FUSED_B. The workspace is
 * spec_workspace_bytes(B, K, V, dtype, 0) bytes.
 * Errors: host-side argument errors return without launching. On the
 * device, a sequence that fails the check (invalid temperature, draft id
 * or logits) sets SPEC_EDEVICE, accept_len = -1 and out_tok = -1 for it, and
 * then nothing is committed; a commit that fails its checks sets
 * SPEC_EINVAL or SPEC_ENOBLOCKS and changes no table, length, stack entry,
 * pool slot, hidden row or offset, while the verification outputs stand.
 * ------------------------------------------------------------------------- */
int spec_verify_chain_commit(const void* tgt, int64_t ld_tgt, const void* drf,
                             int64_t ld_drf, int dtype, int B, int K, int V,
                             const int32_t* draft_tok, const float* temperature,
                             uint64_t seed, const int32_t* seq_id, uint32_t round,
                             int32_t* accept_len, int32_t* out_tok, double* diag,
                             int block_size, int max_blocks, int32_t* block_tables,
                             int32_t* seq_lens, const int32_t* base_len,
                             int32_t* free_stack, int32_t* free_top, int num_blocks,
                             const void* kv_stage, void* kv_pool, int layers,
                             int kv_heads, int head_dim, const void* hid_stage,
                             void* hid_out, int32_t* hid_off, int hidden,
                             int32_t* dev_status, void* ws, size_t ws_bytes,
                             void* stream);

/* The second half of spec_verify_chain_commit (its last two launches), for
 * callers that time or schedule the row statistics apart: the workspace,
 * logits and temperatures must be those of the preceding
 * spec_chain_row_stats call on the same stream (which also clears the
 * workspace word this call's accept launch counts finished sequences in).
 * Arguments, results and errors as for spec_verify_chain_commit. */
int spec_chain_decide_commit(const void* tgt, int64_t ld_tgt, const void* drf,
                             int64_t ld_drf, int dtype, int B, int K, int V,
                             const int32_t* draft_tok, const float* temperature,
                             uint64_t seed, const int32_t* seq_id, uint32_t round,
                             int32_t* accept_len, int32_t* out_tok, double* diag,
                             int block_size, int max_blocks, int32_t* block_tables,
                             int32_t* seq_lens, const int32_t* base_len,
                             int32_t* free_stack, int32_t* free_top, int num_blocks,
                             const void* kv_stage, void* kv_pool, int layers,
                             int kv_heads, int head_dim, const void* hid_stage,
                             void* hid_out, int32_t* hid_off, int hidden,
                             int32_t* dev_status, void* ws, size_t ws_bytes,
                             void* stream);

/* ---------------------------------------------------------------------------
 * The same two calls on one persistent kernel ([HS] "Verlustfreie Garantie",
 * "Wiederverwendung von KV-Cache", "Unterstuetzung fuer Batch-Inferenz", as
 * above). A prologue launch clears the call's counters in the workspace, then
 * one CTA of 16 warps per SM takes (row, chunk) items of the logit rows from
 * a counter in global memory (dynamic balance over the SMs); the warp that
 * completes a row combines it, the one that completes a sequence runs its
 * accept test, residual draws run as 4 KiB parts of the row pair taken by
 * any warp, and (the commit form) the warp that checks the last sequence
 * plans the commit before every warp copies 8 KiB units of the kept rows.
 * Arguments, layouts, results and errors: those of spec_verify_chain and
 * spec_verify_chain_commit (same workspace size); a bounded wait that runs
 * out records SPEC_ETIMEOUT and stops every other wait of the call. The
 * outputs agree with the other entry points' to the verification tolerance
 * (the row sums are taken in chunks of other sizes, so bits may differ).
 * ------------------------------------------------------------------------- */
int spec_verify_chain_persistent(const void* tgt, int64_t ld_tgt, const void* drf,
                                 int64_t ld_drf, int dtype, int B, int K, int V,
                                 const int32_t* draft_tok, const float* temperature,
                                 uint64_t seed, const int32_t* seq_id, uint32_t round,
                                 int32_t* accept_len, int32_t* out_tok, double* diag,
                                 int32_t* dev_status, void* ws, size_t ws_bytes,
                                 void* stream);
int spec_verify_chain_commit_persistent(
    const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype, int B, int K,
    int V, const int32_t* draft_tok, const float* temperature, uint64_t seed,
    const int32_t* seq_id, uint32_t round, int32_t* accept_len, int32_t* out_tok, double* diag,
    int block_size, int max_blocks, int32_t* block_tables, int32_t* seq_lens,
    const int32_t* base_len, int32_t* free_stack, int32_t* free_top, int num_blocks,
    const void* kv_stage, void* kv_pool, int layers, int kv_heads, int head_dim,
    const void* hid_stage, void* hid_out, int32_t* hid_off, int hidden, int32_t* dev_status,
    void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Draft step ([HS] Kernmechanismus: the shallow exit L_d drafts the tokens the
 * deeper exits check; [SV] the entropy of the drafting distribution). The
 * pages print no interface; this is the step that produces the draft_tok of
 * the verification calls, one slot per sequence.
 *
 * logits : drafting-exit rows [B, V]; row b starts at element b * ld.
 * dtype  : SPEC_F32 or SPEC_BF16.
 * temperature : float [B]: 0 (greedy: argmax, smallest id on ties) or within
 *               [1e-6, 1e6]; anything else marks the row invalid.
 * seed, seq_id (int32 [B]), round, pos (int32 [B]) : Philox counter
 *               (seq_id[b], round, pos[b], 0); its lane 1 drives the draw,
 *               pos[b] being the slot the drafted token will occupy.
 * out_tok     : out int32 [B]: the smallest v with sum_{t<=v} q_t > u * sum_t
 *               q_t, q = softmax(l / T) (the argmax for T == 0); -1 for an
 *               invalid row.
 * out_logq    : optional out double [B] (NULL to skip): ln q(out_tok); 0 for
 *               greedy rows, NaN for invalid ones.
 * out_entropy : optional out double [B] (NULL to skip): -sum_v q_v ln q_v in
 *               nats; 0 for greedy rows, NaN for invalid ones.
 * dev_status  : SPEC_EDEVICE for an invalid temperature or a row without a
 *               finite maximum.
 * ws, ws_bytes: spec_draft_workspace_bytes(B, V, dtype) bytes, 256-byte
 *               aligned. No initial contents are needed.
 * One launch when a row fits the shared memory of a cluster of 8 CTAs
 * (V * element size up to about 790 KiB; the workspace is then unused), else two.
 * ------------------------------------------------------------------------- */
size_t spec_draft_workspace_bytes(int B, int V, int dtype);
int spec_draft_sample(const void* logits, int64_t ld, int dtype, int B, int V,
                      const float* temperature, uint64_t seed,
                      const int32_t* seq_id, uint32_t round, const int32_t* pos,
                      int32_t* out_tok, double* out_logq, double* out_entropy,
                      int32_t* dev_status, void* ws, size_t ws_bytes,
                      void* stream);

/* ---------------------------------------------------------------------------
 * Outcome law of a chain check with the drafts fixed ([SSD] Technische
 * Zusammenfassung 2: predict the running verification's outcome, accepted
 * count and bonus token, and prepare continuations for the likely ones; 3.A:
 * a budget spent mostly on short acceptance lengths; 3.B: the token after a
 * rejection follows the residual). The pages print no interface.
 *
 * Same logits, dtype, sizes, drafts and temperatures as spec_verify_chain.
 * With beta_j = min(1, p_j(x_j) / q_j(x_j)) (at T == 0: 1 iff x_j is the
 * argmax of target row j):
 * p_len   : out double [B, K+1]: P(a = k) = beta_0..beta_{k-1} (1 - beta_k)
 *           for k < K, beta_0..beta_{K-1} for k = K.
 * beta    : optional out double [B, K] (NULL to skip).
 * mass    : optional out double [B, K+1]: sum_v max(0, p_k - q_k) for k < K,
 *           1 for k = K (and for greedy sequences).
 * n_top   : outcomes kept per sequence, 0 .. SPEC_MAX_TOP.
 * top_len, top_tok, top_prob : out [B, n_top] (int32, int32, double): the
 *           n_top most likely outcomes (k, v) by P(a = k) r_k(v), most likely
 *           first, equal probabilities in (k, v) order, where r_k =
 *           normalize(max(0, p_k - q_k)) for k < K, r_K = p_K (greedy: the
 *           point mass on the argmax). Entries past the last outcome of
 *           nonzero probability hold -1, -1, 0.
 * dev_status : SPEC_EDEVICE for an invalid temperature, a draft id outside
 *           [0, V) or a row without a finite maximum (outputs NaN / -1).
 * ws, ws_bytes : spec_outcome_workspace_bytes(B, K, V, dtype, n_top) bytes,
 *           256-byte aligned. No initial contents are needed.
 * ------------------------------------------------------------------------- */
size_t spec_outcome_workspace_bytes(int B, int K, int V, int dtype, int n_top);
int spec_outcome_law(const void* tgt, int64_t ld_tgt, const void* drf,
                     int64_t ld_drf, int dtype, int B, int K, int V,
                     const int32_t* draft_tok, const float* temperature,
                     int n_top, double* p_len, double* beta, double* mass,
                     int32_t* top_len, int32_t* top_tok, double* top_prob,
                     int32_t* dev_status, void* ws, size_t ws_bytes,
                     void* stream);

/* ---------------------------------------------------------------------------
 * Chain verification without a caller workspace. The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory where they verify (a fixed memory budget, an allocator owned
 * by a host program, a loop that must not call an allocator). It does what
 * spec_verify_chain does, with the same arguments minus the workspace, and
 * takes its scratch from an array of SPEC_NOALLOC_SCRATCH_BYTES compiled into
 * the library; every GPU that loads the library holds that array until the
 * process exits. It calls no allocating routine.
 *   - Sizes whose workspace (spec_workspace_bytes(B, K, V, dtype, 0)) would
 *     exceed the array return SPEC_EWORKSPACE and launch nothing.
 *   - A call looks the array's device address up with the device current
 *     (cudaGetSymbolAddress) and keeps it per device and CUDA context, so the
 *     lookup runs on the first call on a device (and again only after that
 *     device's context was destroyed and re-created); make that first call
 *     outside any stream capture. A failed lookup returns SPEC_ECUDA (text
 *     from spec_last_cuda_error) and is not kept: the next call retries.
 *   - All calls share the one array and it keeps the previous call's
 *     contents (no call reads what an earlier one left). Calls that overlap
 *     on the GPU (several streams or threads) race on it and must not be made.
 * ------------------------------------------------------------------------- */
#define SPEC_NOALLOC_SCRATCH_BYTES (16u << 20)
int spec_verify_chain_noalloc(const void* tgt, int64_t ld_tgt, const void* drf,
                              int64_t ld_drf, int dtype, int B, int K, int V,
                              const int32_t* draft_tok, const float* temperature,
                              uint64_t seed, const int32_t* seq_id, uint32_t round,
                              int32_t* accept_len, int32_t* out_tok, double* diag,
                              int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Saguaro sampling ([SSD] Technische Zusammenfassung 3.B): lower the draft
 * probability of the tokens held in the speculation cache, so a rejection's
 * residual (proportional to the target-minus-draft difference) lands on them
 * more often. The lowered draft law is q'(v) proportional to
 * q(v) (1 - eps [v cached]); at temperature T > 0 that is the softmax of the
 * draft logits with T ln(1 - eps) added to the cached tokens, which this call
 * adds IN PLACE to every draft row of each sequence. Run it on the drafting
 * exit's rows before spec_draft_sample and the verification: both then use
 * q' as the draft law and the check stays lossless.
 *
 * logits      : draft rows [B, rows_per_seq, V] (in/out); row (b, r) starts
 *               at element (b * rows_per_seq + r) * ld. The rows of a chain
 *               check are [B, K, V] (rows_per_seq = K); those of the draft
 *               step [B, V] (rows_per_seq = 1).
 * dtype       : SPEC_F32 or SPEC_BF16. The shift float32(T * ln(1 - eps))
 *               is added in float32 and the sum rounded to the rows' type.
 * cached      : int32 token ids, [B, n_cached] (per_row = 0: one list per
 *               sequence, lowered in each of its rows) or
 *               [B, rows_per_seq, n_cached] (per_row = 1: one list per row,
 *               e.g. the bonus tokens prepared for that position). Ids
 *               outside [0, V) are padding; an id repeated within a list is
 *               lowered once.
 * n_cached    : 0 .. SPEC_MAX_CACHED ids per list.
 * per_row     : 0 or 1, as above.
 * eps         : the lowering, 0 <= eps < 1 (0: nothing to do).
 * temperature : float [B]; sequences at 0 (greedy) or with an invalid
 *               temperature are left unchanged.
 * Returns SPEC_EINVAL for bad sizes, dtype, per_row or eps (nothing
 * launched); SPEC_ECUDA if the launch fails.
 * ------------------------------------------------------------------------- */
int spec_saguaro_adjust(void* logits, int64_t ld, int dtype, int B, int rows_per_seq, int V,
                        const int32_t* cached, int n_cached, int per_row, double eps,
                        const float* temperature, void* stream);

/* ---------------------------------------------------------------------------
 * Vocabulary-parallel chain verification. The check of spec_verify_chain
 * (speculative sampling as HiSpec, gist.science summary of arXiv 2510.01336,
 * section 2 "Verlustfreie Garantie", appeals to it; residual per Speculative
 * Speculative Decoding, Technische Zusammenfassung 3.B) for rows split over
 * the vocabulary: rank r of R holds the columns [v0, v0 + Vs) of every target
 * and draft row (e.g. the output of a vocabulary-parallel LM head) and no
 * rank ever holds a whole row. The partition functions, greedy argmaxes and
 * residual masses are sums or maxima over the vocabulary, so the ranks
 * exchange small records instead of rows. Per call, on every rank in the same
 * order (the exchanges are the caller's collectives, e.g. NCCL):
 *
 *   spec_vp_shard_stats -> rows_out [B, 2K+1] records
 *   all-gather rows_out in rank order       -> rows_all [R, B, 2K+1]
 *   spec_vp_decide      -> mass_out [B]     (every rank: same accepted counts)
 *   all-gather mass_out in rank order       -> mass_all [R, B]
 *   spec_vp_pick        -> accept_len [B], out_tok [B, K+1] (-1 at the drawn
 *                          position unless this rank drew it), diag
 *   max-reduce out_tok over the ranks       -> the tokens of spec_verify_chain
 *
 * The outputs follow spec_verify_chain's rule on the same Philox counters;
 * they differ from a one-GPU call only where the order of the sums moves a
 * decision (fp64 margin below 1e-6). The records are opaque bytes
 * (SPEC_VP_ROW_BYTES, SPEC_VP_MASS_BYTES each, 8-byte aligned).
 *
 * Common arguments:
 * tgt, ld_tgt : this rank's target columns [B, K+1, Vs], row stride ld_tgt
 *               >= Vs elements; rows 16-byte aligned.
 * drf, ld_drf : its draft columns [B, K, Vs] (may be NULL when K == 0).
 * Vs, v0, V   : the shard [v0, v0 + Vs) of the vocabulary [0, V); the R
 *               shards must cover [0, V) without overlap (a drafted id that
 *               no shard holds flags the sequence).
 * R, rank     : 1 <= R <= SPEC_VP_MAX_RANKS, 0 <= rank < R.
 * draft_tok, temperature, seed, seq_id, round, diag: as spec_verify_chain;
 *               diag is written identically by every rank.
 * ws          : spec_vp_workspace_bytes(B, K, Vs, dtype) bytes, 256-byte
 *               aligned, kept by the caller from spec_vp_shard_stats through
 *               spec_vp_pick of the same call.
 * Errors: SPEC_EINVAL / SPEC_EWORKSPACE on the host before any launch;
 * sequences with invalid values get accept_len = -1, out_tok = -1 and
 * SPEC_EDEVICE in dev_status on every rank alike.
 * ------------------------------------------------------------------------- */
size_t spec_vp_workspace_bytes(int B, int K, int Vs, int dtype);
int spec_vp_shard_stats(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                        int dtype, int B, int K, int Vs, int v0, int V,
                        const int32_t* draft_tok, const float* temperature, void* rows_out,
                        int32_t* dev_status, void* ws, size_t ws_bytes, void* stream);
int spec_vp_decide(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                   int B, int K, int Vs, int v0, int V, int R, int rank, const void* rows_all,
                   const int32_t* draft_tok, const float* temperature, uint64_t seed,
                   const int32_t* seq_id, uint32_t round, void* mass_out, double* diag,
                   int32_t* dev_status, void* ws, size_t ws_bytes, void* stream);
int spec_vp_pick(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                 int B, int K, int Vs, int v0, int V, int R, int rank, const void* mass_all,
                 const int32_t* draft_tok, const float* temperature, int32_t* accept_len,
                 int32_t* out_tok, double* diag, int32_t* dev_status, void* ws, size_t ws_bytes,
                 void* stream);

/* Test hook (no counterpart in the paper): the limit of the row-statistics
 * kernel's waits for its tile copies on the current device, in nanoseconds
 * (2e9 by default). 0 makes every such wait one non-blocking test, so a copy
 * still in flight makes it run out: the kernel then records SPEC_ETIMEOUT in
 * dev_status, waits (2 s at most) for its copies in flight and returns; a
 * commit in the same call changes nothing. Lets a test exercise the timeout
 * path without any hang; set it back to 2000000000 afterwards. It is a
 * device-wide setting: calls on other streams see it too. */
int spec_test_set_wait_limit_ns(uint64_t ns);

/* Test hook (no counterpart in the paper): the limit of the wait, in
 * nanoseconds (2e9 by default), of spec_verify_chain_commit's copy launch for
 * the plan word that its decide launch's planner sets. 0 makes the wait one
 * poll, so copy CTAs that start before the plan is written run out: they
 * record SPEC_ETIMEOUT in dev_status and copy nothing. The verification
 * outputs stand; the plan is made in full, or not at all when the timeout is
 * recorded before the planner reads the status word; kept rows may be left
 * uncopied. Set it
 * back to 2000000000 afterwards; a device-wide setting, as above. */
int spec_test_set_copy_wait_limit_ns(uint64_t ns);

/* Test hook of spec_verify_chain_noalloc (no counterpart in the paper):
 * forgets every kept scratch address and makes the next n address lookups
 * fail as a lookup inside a stream capture does (SPEC_ECUDA), so a test can
 * check that a failed lookup does not stay cached. n >= 0; 0 ends it. */
int spec_noalloc_test_fail_lookups(int n);

/* Diagnostic: text of the last CUDA error behind a SPEC_ECUDA return on the
 * calling thread ("no error" if none). Static storage. */
const char* spec_last_cuda_error(void);

/* Diagnostic: the device Philox. For i < n, counter = ctr[4i .. 4i+3]
 * (device uint32), key from `seed`; writes the two uniforms (accept lane,
 * draw lane) to out[2i], out[2i+1] (device float). */
int spec_philox_uniforms(uint64_t seed, const uint32_t* ctr, int n,
                         float* out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SPEC_VERIFY_H */
