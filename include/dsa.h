/*
 * dsa.h -- C ABI of the DeepSeek Sparse Attention (DSA) hot path, B200 (sm_100a).
 *
 * The operations (page "Paper Breakdown: DeepSeek-V3.2", section 2
 * "Architecture: DSA (2.1)"):
 *
 *   index score   I_{t,s} = sum_{j<H_I} w_{t,j} * ReLU(q^I_{t,j} . k^I_s)
 *   selector      the k candidates s <= pos[t] with the largest I_{t,s}
 *                 ("Top-k selector on I_{t,s}"; past tokens only, per the
 *                 summary page "DeepSeek V3.2: Sparse Attention and
 *                 Reinforcement Learning Updates"; k = 2048 per the research
 *                 summary's "Key points")
 *   attention     u_t = Attn(h_t, {c_s : s selected}), MLA in MQA mode: every
 *                 query head attends to the same latent row c_s
 *                 ("DSA under MLA (MQA Mode)").
 *
 * Conventions shared by every entry point
 *  - Pointers are DEVICE pointers owned by the caller. The library keeps no
 *    pointer after a call returns and allocates no device memory: scratch
 *    comes from the caller's `workspace`. `stream` is a cudaStream_t (NULL =
 *    legacy default stream); every call is asynchronous on it.
 *  - Tensors are dense and row-major. FP8 tensors hold OCP E4M3 bytes; BF16
 *    tensors hold bfloat16 values. Every pointer must be 16-byte aligned.
 *  - Query row t sees the candidates s = 0..pos[t] of its own sequence, whose
 *    key/latent rows sit at k_base[t] + s in the caches. pos == NULL means
 *    pos[t] = t + S - T (one causal sequence whose last T rows are the
 *    queries); k_base == NULL means k_base[t] = 0. k_base[t] + pos[t] < S.
 *  - Return value: DSA_OK, or a negative dsa_status. Arguments are checked
 *    before any launch; nothing is launched when a check fails. The message of
 *    the last failure on the calling thread is dsa_last_error().
 *  - Kernels that wait on on-chip barriers bound every wait; a wait that runs
 *    out records DSA_ERR_TIMEOUT in a device status word read (and cleared)
 *    by dsa_device_status().
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_ARG = -1,         /* NULL pointer, size <= 0, misaligned pointer, bad pos/k_base */
    DSA_ERR_UNSUPPORTED = -2, /* a dimension outside the supported set (below) */
    DSA_ERR_CUDA = -3,        /* a CUDA runtime error at launch (or an earlier asynchronous one) */
    DSA_ERR_TIMEOUT = -4,     /* a kernel gave up a bounded wait (see dsa_device_status) */
    DSA_ERR_WORKSPACE = -5,   /* workspace NULL or smaller than dsa_workspace_size() */
    DSA_ERR_CHECK = -6        /* debug build only: a device check counted invalid index-set entries */
} dsa_status;

/*
 * Bytes of device workspace that dsa_indexer_topk, dsa_sparse_mla_attn and
 * dsa_forward need for these sizes (the maximum over the three). 0 is a valid
 * answer; a NULL workspace is then accepted. The workspace is scratch: its
 * contents on entry do not matter and are undefined on return. Two calls in
 * flight at the same time need two workspaces.
 */
size_t dsa_workspace_size(int T, int S, int H_I, int d_I, int k, int Hq, int d_qk, int d_v);

/*
 * Lightning indexer + Top-k selector ("Index score" and "Top-k selector",
 * section 2 of "Paper Breakdown: DeepSeek-V3.2").
 *
 *   q_idx   e4m3 [T, H_I, d_I]   indexer query heads
 *   w       fp32 [T, H_I]        head weights
 *   k_idx   e4m3 [S, d_I]        indexer keys
 *   pos     int32 [T] or NULL    last candidate of each row (see above)
 *   k_base  int32 [T] or NULL    first cache row of each row's sequence
 *   k       number of selected entries per row
 *   idx     int32 [T, k] (out)   row t: the min(k, pos[t]+1) selected s values
 *                                (relative to k_base[t]), distinct, in
 *                                unspecified order, followed by -1 padding.
 *
 * Scores are formed in fp32 (FP8 products are exact in fp32). Among equal
 * scores the lower s is selected first, so the result is unique.
 * Supported: H_I <= 16, d_I in {32, 64, 128, 256}, 1 <= k <= 4096; with pos
 * or k_base given, or H_I != 8, or d_I != 128, S <= 2^27 (DSA_ERR_UNSUPPORTED
 * beyond, before any launch).
 */
int dsa_indexer_topk(const void* q_idx, const float* w, const void* k_idx, const int32_t* pos,
                     const int32_t* k_base, int T, int S, int H_I, int d_I, int k, int32_t* idx,
                     void* workspace, size_t ws_bytes, void* stream);

/*
 * Indexer + Top-k for a batch of packed causal sequences (variable-length
 * prefill; the serving form of dsa_indexer_topk, no counterpart on the pages
 * beyond the per-sequence definition).
 *
 *   cu_q   int32 [n_seqs+1], HOST memory: sequence b owns query rows
 *          [cu_q[b], cu_q[b+1]) of q_idx, w and idx
 *   cu_k   int32 [n_seqs+1], HOST memory: sequence b owns key rows
 *          [cu_k[b], cu_k[b+1]) of k_idx
 *
 * Each sequence is a suffix-aligned causal prefill: its j-th query row sees
 * keys s <= j + (S_b - T_b) of its own keys (T_b <= S_b), and idx values are
 * relative to cu_k[b]. Equivalent to dsa_indexer_topk with
 * pos[t] = j + S_b - T_b and k_base[t] = cu_k[b], but each sequence runs the
 * streaming tensor-core path. cu_q[0] = cu_k[0] = 0; cu_q[b] * H_I * 4 and
 * cu_q[b] * k * 4 must be multiples of 16 (always so for H_I = 8 and k % 4 ==
 * 0). Workspace: dsa_workspace_size(max_b T_b, max_b S_b, ...) suffices.
 * Sequences run one after another on `stream`.
 */
int dsa_indexer_topk_varlen(const void* q_idx, const float* w, const void* k_idx, const int32_t* cu_q,
                            const int32_t* cu_k, int n_seqs, int H_I, int d_I, int k, int32_t* idx,
                            void* workspace, size_t ws_bytes, void* stream);

/*
 * Paged caches (the serving form of the decode path; the method itself is
 * defined per sequence). A sequence's cache rows are pages of page_size rows
 * (a multiple of 64) in a pool of num_pages pages:
 *
 *   block_table int32 [n_seqs, max_pages] (device): entry [b, j] is the pool
 *               page holding logical keys [j*page_size, (j+1)*page_size) of
 *               sequence b
 *   seq         int32 [T] (device): the sequence of query row t
 *   pos         int32 [T] (device): the last logical key row t sees
 *
 * idx values are logical positions within the row's sequence. Block-table
 * entries outside [0, num_pages) are read as page 0 (no access outside the
 * pool, wrong values); a row whose seq is outside [0, n_seqs) has no keys.
 *
 * dsa_indexer_topk_paged: k_pages e4m3 [num_pages * page_size, d_I], d_I = 128
 * (H_I <= 16, k as dsa_indexer_topk); workspace as dsa_workspace_size(T,
 * max_pages * page_size, ...).
 */
int dsa_indexer_topk_paged(const void* q_idx, const float* w, const void* k_pages, int num_pages,
                           int page_size, const int32_t* block_table, int n_seqs, int max_pages,
                           const int32_t* seq, const int32_t* pos, int T, int H_I, int d_I, int k,
                           int32_t* idx, void* workspace, size_t ws_bytes, void* stream);

/*
 * dsa_sparse_mla_attn over a paged latent cache: kv_pages bf16
 * [num_pages * page_size, d_qk]; Hq = 128, d_qk = 576, d_v = 512 (other
 * arguments as dsa_sparse_mla_attn; no workspace).
 */
int dsa_sparse_mla_attn_paged(const void* q, const void* kv_pages, int num_pages, int page_size,
                              const int32_t* block_table, int n_seqs, int max_pages, const int32_t* seq,
                              const int32_t* pos, const int32_t* idx, int T, int Hq, int d_qk, int d_v,
                              int k, float scale, void* out, float* lse, void* stream);

/*
 * Sparse MQA attention over the selected latent rows ("Attention" and "DSA
 * under MLA (MQA Mode)", section 2 of "Paper Breakdown: DeepSeek-V3.2").
 *
 *   q      bf16 [T, Hq, d_qk]   query heads (latent + rope parts)
 *   kv     bf16 [S, d_qk]       latent rows c_s; the value is c_s[0:d_v]
 *   idx    int32 [T, k]         selected s per row (relative to k_base[t]).
 *                               Entries < 0 or > pos[t] are ignored. Valid
 *                               entries come first: the call reads only the
 *                               first min(k, pos[t]+1) entries of a row.
 *   scale  softmax scale (e.g. 1/sqrt(d_qk))
 *   out    bf16 [T, Hq, d_v] (out)   sum_s softmax_s(scale q.c_s) c_s[0:d_v]
 *   lse    fp32 [T, Hq] (out)        log sum_s exp(scale q.c_s) (natural log);
 *                                    -inf and out = 0 for a row with no entry
 * Supported: Hq <= 1024, d_v <= d_qk <= 1024, d_v even, d_qk % 8 == 0,
 * 1 <= k <= 4096.
 */
int dsa_sparse_mla_attn(const void* q, const void* kv, const int32_t* idx, const int32_t* pos,
                        const int32_t* k_base, int T, int S, int Hq, int d_qk, int d_v, int k,
                        float scale, void* out, float* lse, void* workspace, size_t ws_bytes,
                        void* stream);

/*
 * dsa_sparse_mla_attn with the number of parts each row's selected set is
 * split into chosen by the caller (the decode form: one query token per
 * sequence, so few rows must fill the GPU). The row's valid entries are cut
 * into `splits` contiguous ranges of whole 64-entry chunks; each range is
 * attended by its own CTAs, which write the part's output normalised by its
 * own softmax sum and its log-sum-exp, and a merge kernel combines the parts:
 *   lse = log sum_z exp(lse_z),   out = sum_z exp(lse_z - lse) out_z
 * (the split of the selected set across CTAs with a log-sum-exp merge:
 * "DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models",
 * "2.3 Inference Costs"). splits = 0 is the library's own choice (what
 * dsa_sparse_mla_attn uses: parts only where they add no wave of work);
 * 1..16 forces that many (a part may be empty). The result equals the
 * unsplit one up to fp32 rounding of the merge.
 * workspace: dsa_sparse_mla_attn_split_workspace_size(T, Hq, d_v, splits)
 * bytes (0 for splits = 1; for splits = 0 use dsa_workspace_size).
 * Other arguments and limits as dsa_sparse_mla_attn; DSA_ERR_ARG for splits
 * outside 0..16.
 */
size_t dsa_sparse_mla_attn_split_workspace_size(int T, int Hq, int d_v, int splits);
int dsa_sparse_mla_attn_split(const void* q, const void* kv, const int32_t* idx, const int32_t* pos,
                              const int32_t* k_base, int T, int S, int Hq, int d_qk, int d_v, int k, float scale,
                              int splits, void* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * Backward of dsa_sparse_mla_attn: the gradients through the selected latent
 * rows only, as the sparse training stage trains the main model ("Paper
 * Breakdown: DeepSeek-V3.2", table "Continued Pre-Training (2.1.1)", row
 * "Sparse Training"). With p_s = exp(scale q_h.c_s - lse_h) over row t's
 * valid entries, dp_s = dout_h.c_s[0:d_v] and D_h = dout_h.out_h:
 *   dq[t,h]        = scale sum_s p_s (dp_s - D_h) c_s
 *   dkv[base + s] += scale sum_h p_s (dp_s - D_h) q_h + sum_h p_s dout_h
 *                    (the second term on the first d_v columns only)
 * Inputs as dsa_sparse_mla_attn, plus the forward's results for the same
 * idx:
 *   out    bf16 [T, Hq, d_v]   forward output (gives D_h)
 *   lse    fp32 [T, Hq]        forward log-sum-exp
 *   dout   bf16 [T, Hq, d_v]   gradient of the loss with respect to out
 * Outputs (device memory, caller-owned):
 *   dq     fp32 [T, Hq, d_qk]  written in full
 *   dkv    fp32 [S, d_qk]      ACCUMULATED into (atomic adds, so the order of
 *                              the adds and the last bits vary run to run);
 *                              zero it for a fresh gradient
 * workspace: at least one row of scratch (dsa_sparse_mla_attn_bwd_workspace_size
 * with T = 1); more lets the call take more rows per pass (up to 8192 per
 * pass, DSA_ERR_WORKSPACE below one row). Rows are processed in passes of
 * that many rows on `stream`; the workspace holds the bf16 scale*dz of one
 * pass between its kernels, and each row's per-head dO.O.
 * Supported: Hq <= 128, d_qk % 16 == 0, d_qk <= 576, d_v % 16 == 0,
 * d_v <= d_qk, 1 <= k <= 4096 (DSA_ERR_UNSUPPORTED otherwise).
 */
size_t dsa_sparse_mla_attn_bwd_workspace_size(int T, int Hq, int k);
int dsa_sparse_mla_attn_bwd(const void* q, const void* kv, const int32_t* idx, const int32_t* pos,
                            const int32_t* k_base, const void* out, const float* lse, const void* dout,
                            int T, int S, int Hq, int d_qk, int d_v, int k, float scale, float* dq,
                            float* dkv, void* workspace, size_t ws_bytes, void* stream);

/*
 * Indexer KL loss over each row's selected set and its gradient with respect
 * to the indexer's inputs: the objective that trains the lightning indexer
 * toward the main attention ("Paper Breakdown: DeepSeek-V3.2", table
 * "Continued Pre-Training (2.1.1)": dense warm-up L^I = sum_t
 * D_KL(p_{t,:} || Softmax(I_{t,:})) with the main model frozen; sparse stage:
 * the same KL over the selected set S_t, indexer input detached). The pages
 * leave p_{t,:} undefined; here it is the main attention of row t summed over
 * the query heads and L1-normalised over S_t:
 *   p_s  = sum_h exp(scale q_h.c_s - lse_h) / (sum over s' in S_t and h)
 *   I_s  = sum_j w_j ReLU(q^I_j.k^I_s)          (unrounded fp32)
 *   loss[t] = sum_{s in S_t} p_s (log p_s - log softmax_{S_t}(I)_s)
 * and, with dI_s = softmax_{S_t}(I)_s - p_s (p is a constant):
 *   dw[t,j]       = sum_s dI_s ReLU(q^I_j.k^I_s)
 *   dq_idx[t,j,:] = sum_s dI_s w_j [q^I_j.k^I_s > 0] k^I_s
 *   dk_idx[s,:]  += sum_t sum_j dI_s w_j [q^I_j.k^I_s > 0] q^I_j
 * S_t is row t's idx entries (valid entries first; only the first
 * min(k, pos[t]+1) are read, negatives and entries > pos[t] ignored). The
 * dense warm-up loss is this call with every s <= pos[t] in idx (k >= L).
 * Inputs: q, kv, idx, pos, k_base, scale as dsa_sparse_mla_attn; lse fp32
 * [T, Hq] its log-sum-exp for the same idx; q_idx, w, k_idx as
 * dsa_indexer_topk (e4m3, fp32, e4m3).
 * Outputs (device, caller-owned): loss fp32 [T]; dw fp32 [T, H_I]; dq_idx
 * fp32 [T, H_I, d_I] (written); dk_idx fp32 [S, d_I] ACCUMULATED (atomic
 * adds; zero it for a fresh gradient). A row without entries gives 0.
 * workspace: at least dsa_indexer_kl_workspace_size(1, k) bytes; up to 8192
 * rows per pass (DSA_ERR_WORKSPACE below one row).
 * Supported: Hq <= 128, d_qk % 16 == 0 and <= 576, H_I <= 16, d_I % 16 == 0
 * and <= 256, H_I * d_I <= 4096, 1 <= k <= 4096 (DSA_ERR_UNSUPPORTED).
 */
size_t dsa_indexer_kl_workspace_size(int T, int k);
int dsa_indexer_kl(const void* q, const void* kv, const int32_t* idx, const int32_t* pos, const int32_t* k_base,
                   const float* lse, const void* q_idx, const float* w, const void* k_idx, int T, int S, int Hq,
                   int d_qk, int H_I, int d_I, int k, float scale, float* loss, float* dw, float* dq_idx,
                   float* dk_idx, void* workspace, size_t ws_bytes, void* stream);

/*
 * MLA in MHA mode over one causal sequence: every head has its own key and
 * value rows (the latent row expanded per head), where the sparse path's MQA
 * mode shares one latent row across heads (the bilingual paper summary's
 * section list, "Appendix A MHA and MQA Modes of MLA", title only; "Paper
 * Breakdown: DeepSeek-V3.2", section 2, "DSA under MLA (MQA Mode)"). On a
 * short prefill (L <= k) the selector keeps every causal key, so this is dense
 * causal attention: for query row t (position pos[t] = t + S - T) and head h,
 *   out[t,h] = sum_{s <= pos[t]} softmax_s(scale q[t,h].k[s,h]) v[s,h]
 *   lse[t,h] = log sum_{s <= pos[t]} exp(scale q[t,h].k[s,h])
 * Arguments (device memory, caller-owned, row-major, 16-byte aligned):
 *   q   bf16 [T, Hq, d_h]     queries of the last T tokens
 *   k   bf16 [S, Hq, d_h]     per-head keys of all S tokens
 *   v   bf16 [S, Hq, d_hv]    per-head values
 *   out bf16 [T, Hq, d_hv] (out), lse fp32 [T, Hq] (out, natural log)
 * Supported: (d_h, d_hv) in {(192, 128), (64, 64)}, 0 < T <= S, Hq <= 65535.
 * Asynchronous on `stream`; no workspace.
 */
int dsa_mla_mha_attn(const void* q, const void* k, const void* v, int T, int S, int Hq, int d_h, int d_hv,
                     float scale, void* out, float* lse, void* stream);

/*
 * The whole hot path: dsa_indexer_topk followed by dsa_sparse_mla_attn on the
 * same stream. `idx` is an output the caller keeps (it is also the input of
 * the attention step). Argument meanings and limits as above.
 */
int dsa_forward(const void* q_idx, const float* w, const void* k_idx, const void* q,
                const void* kv, const int32_t* pos, const int32_t* k_base, int T, int S, int H_I,
                int d_I, int Hq, int d_qk, int d_v, int k, float scale, int32_t* idx, void* out,
                float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * dsa_indexer_topk without a workspace argument. The paper has no
 * counterpart: this entry point exists for callers that cannot give the
 * library device memory -- code that must not call cudaMalloc (whose implicit
 * device synchronisation can stall other work, or which a host framework's
 * memory pool forbids) and has no spare buffer of its own to lend.
 *
 * Same arguments, result and limits as dsa_indexer_topk, minus the workspace;
 * it allocates nothing. Its scratch is a 16 MiB array (4,194,304 fp32 scores)
 * that the library holds in the device memory of every GPU it is loaded on,
 * until the process exits. Calls with S > 4,194,304 are rejected with
 * DSA_ERR_UNSUPPORTED before any launch. The first call on a device looks up
 * the array's device address for that device; make that first call before
 * any stream capture. Every call on a device shares the one array, so calls
 * whose kernels overlap on the GPU (two streams, two host threads) race and
 * must be serialised by the caller; nothing in the array has to start at
 * zero, and it keeps whatever the last call wrote.
 */
int dsa_indexer_topk_noalloc(const void* q_idx, const float* w, const void* k_idx,
                             const int32_t* pos, const int32_t* k_base, int T, int S, int H_I,
                             int d_I, int k, int32_t* idx, void* stream);

/*
 * Multi-GPU partition (host-only; no device memory, no launch). The path
 * shards with no exchange between ranks: query rows of one causal prefill
 * are independent once every rank holds the key and latent caches, and
 * decode sequences are independent altogether. These functions give rank r
 * the contiguous range [bounds[r], bounds[r+1]) with about equal modelled
 * work (bounds: caller-owned HOST int32 [parts + 1]; bounds[0] = 0,
 * bounds[parts] = the item count; a range may be empty when parts exceeds
 * the items).
 *
 * dsa_partition_prefill_rows: the T query rows of one causal sequence of S
 * tokens (row t at position t + S - T). Row cost: when it has n > k
 * candidates, the indexer's n (row, key) pairs at 2 H_I d_I FP8 flop each,
 * counted at half weight (FP8 runs at twice the BF16 rate; rows with n <= k
 * need no scores), plus min(n, k) selected rows at 2 Hq (d_qk + d_v) BF16
 * flop each. The causal cost grows with t (the indexer's O(L^2) term: "Paper
 * Breakdown: DeepSeek-V3.2", "Efficiency (Fig 3)"), so the ranges shrink
 * toward the end of the sequence. A rank runs its rows [t0, t1) as the tail
 * prefill of the first t1 + S - T tokens: dsa_forward with T' = t1 - t0,
 * S' = t1 + S - T, pos = k_base = NULL and the row slices of q_idx, w, q, idx,
 * out and lse; the results equal the one-call results bit for bit.
 *
 * dsa_partition_decode_seqs: n_seqs decode sequences with context lengths
 * ctx (HOST int32 [n_seqs]); cost = ctx d_I key bytes + min(ctx, k) 2 d_qk
 * gathered bytes.
 *
 * DSA_ERR_ARG for NULL pointers or sizes out of range (T <= 0, S < T,
 * parts <= 0, a negative ctx).
 */
int dsa_partition_prefill_rows(int T, int S, int k, int H_I, int d_I, int Hq, int d_qk, int d_v, int parts,
                               int32_t* bounds);
int dsa_partition_decode_seqs(const int32_t* ctx, int n_seqs, int k, int d_I, int d_qk, int parts,
                              int32_t* bounds);

/*
 * Waits for `stream`, then returns and clears the device status word:
 * DSA_OK, DSA_ERR_TIMEOUT (a kernel gave up a bounded wait) or DSA_ERR_CUDA
 * (an asynchronous CUDA error; its text is in dsa_last_error()).
 */
int dsa_device_status(void* stream);

/*
 * Debug build. libdsa_debug.so is the same library compiled with -DDSA_DEBUG
 * (no counterpart in the method: a stand-in for an external memory checker).
 * Every entry point that produces or reads an index set then also validates
 * it on the device, per row t with n = pos[t] + 1 candidates and m =
 * min(k, n) entries read, and counts (never traps):
 *   [0] entries in [0, m) greater than pos[t]   (ignored by the attention)
 *   [1] entries in [0, m) below 0               (ignored by the attention)
 *   [2] valid entries at or past m              (not read by the attention)
 *   [3] repeated valid entries in [0, m)
 *   [4] valid entries whose block-table page is outside the pool (paged calls)
 *   [5] selector results that are not min(k, n) distinct valid entries then -1
 * A call that counts any sets the status word to DSA_ERR_CHECK
 * (dsa_device_status). dsa_debug_build() is 1 in that build, 0 otherwise;
 * dsa_debug_counters copies the first n (<= 6) totals to HOST memory after a
 * device synchronisation and, with reset != 0, clears them. The release build
 * counts nothing (all totals stay 0).
 */
int dsa_debug_build(void);
int dsa_debug_counters(uint64_t* out, int n, int reset);

/*
 * Phase timing (a diagnostic, no counterpart in the method). With
 * dsa_phase_timing(1), every indexer call brackets each of its phases with a
 * pair of CUDA events on its stream: [0] the scores (the sampled and filter
 * scans, or the chunk passes), [1] the threshold (the sampled tau), [2] the
 * Top-k selection (the select or merge kernels). dsa_phase_times copies the
 * first n (<= 3) sums in milliseconds to HOST memory, waiting for the events,
 * and starts new sums. Off by default; when off nothing is recorded.
 */
int dsa_phase_timing(int enable);
int dsa_phase_times(double* ms, int n);

/* Text of the last error on the calling thread ("" when none). */
const char* dsa_last_error(void);

/* ABI version: bumped on any change of a signature or a convention. */
int dsa_abi_version(void);

/*
 * Failure-detection self-test (no counterpart in the method). Launches one
 * warp that waits on a barrier nothing ever signals, with the library's
 * bounded wait shortened to limit_ms (1..2000): the wait gives up, records
 * DSA_ERR_TIMEOUT (barrier tag 999) in the device status word, and the kernel
 * returns; the context stays usable. Returns DSA_OK once the launch is issued
 * (DSA_ERR_ARG for a limit outside 1..2000); read the outcome with
 * dsa_device_status (expected: DSA_ERR_TIMEOUT, then DSA_OK on the next call).
 */
int dsa_selftest_bounded_wait(int limit_ms, void* stream);

/* Number of kernels this process has launched through the library so far
 * (all threads, all devices): a diagnostic for launch accounting. */
uint64_t dsa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
