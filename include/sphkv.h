/*
 * sphkv.h -- C ABI of libsphkv: Spherical KV angle-domain attention (ADA)
 * decode over a paged, tier-homogeneous compressed KV cache, on NVIDIA B200
 * (sm_100a).
 *
 * Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
 * for Efficient Long-Context Inference" (arXiv 2605.18856), Abstract and AI
 * Summary.  ADA stores each key as a scalar radius plus compact angle codes and
 * computes attention logits directly from those codes, with no dense key
 * rebuilt; RDR chooses keep/drop and a precision tier per unit under a fixed
 * byte budget, so that pages are tier-homogeneous and read with coalesced
 * loads.  The pages fix no bit layout; this library fixes the one below.
 *
 * Conventions for every entry point
 *  - All array arguments are DEVICE pointers unless marked "host".  The caller
 *    allocates and owns every buffer; the library allocates nothing.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously; nothing synchronises the host.
 *  - The return value reports host-side argument errors and launch failures.
 *    Problems only the device can see (bad page ids, fp16 overflow, a wait
 *    that ran out) are written to `status_dev` (one device int32, may be NULL):
 *    the kernels store the largest error code seen with an atomic max, so the
 *    caller zeroes it first and reads it after synchronising.
 *  - Head size d is 128 and pages hold 16 tokens.
 *
 * Format
 *  Key k (d = 128) -> radius r = |k| rounded to fp16 (RNE), and the unit
 *  direction in recursive-polar coordinates over a perfect binary tree:
 *   - 64 leaf angles  phi_j = atan2(k[2j+1], k[2j])  (zero pair -> 0), coded on
 *     a periodic grid of 2^b_leaf points c * 2pi / 2^b_leaf;
 *   - 63 upper angles psi = atan2(|right half|, |left half|) in [0, pi/2],
 *     coded on an end-inclusive grid c * (pi/2) / (2^b_up - 1);
 *  rounding to nearest, ties to even, computed in fp64.  Upper nodes are in
 *  level order: level 1 (parents of leaves 2m, 2m+1, m = 0..31), then level 2
 *  (m = 0..15), ..., the root last.
 *  The logit of query q is  r * S_root / sqrt(d), where a leaf gives
 *  S = q[2j] cos(phi) + q[2j+1] sin(phi) and an upper node
 *  S = cos(psi) S_left + sin(psi) S_right.
 *  Value v -> per-token scale s = fp16(max|v| / Q) and codes
 *  clamp(rint(v / s), -Q, Q), Q = 127 (int8) or 7 (int4); s = 0 gives 0 codes.
 *
 *  Tiers: T1 (b_leaf 8, b_up 8, int8 V, 4160 B/page), T2 (4, 6, int4, 2368 B),
 *  T3 (3, 4, int4, 1984 B), or drop (no storage, excluded from the softmax).
 *  Page of tier t, in this order (all fields 16-byte aligned):
 *    r[16] fp16 | vscale[16] fp16 | code planes | value rows [16][16*v_bits]
 *  The sign bit of r is the token's drop flag (see sphkv_set_keep); the
 *  radius itself is the value with that bit cleared.
 *  Codes of a token are regrouped into 8 subtree blocks, block s for leaves
 *  8s..8s+7: L[s][j] = leaf code 8s+j; U[s][0..3] = level-1 nodes 4s..4s+3,
 *  U[s][4..5] = level-2 nodes 2s, 2s+1, U[s][6] = level-3 node s, U[s][7] =
 *  top node s for s < 7 (top nodes: the 4 level-4 nodes, the 2 level-5
 *  nodes, the root), U[7][7] = 0.  Code planes, each [16 tokens][8 blocks]
 *  [width], little-endian:
 *    T1: width 16: bytes 0..7 = L[s][0..7], bytes 8..15 = U[s][0..7];
 *    T2: width 8: u32 nibble j = L[s][j], then the low 32 bits of the
 *        48-bit field F with bits 6j..6j+5 = U[s][j]; width 2: u16 = F >> 32;
 *    T3: width 4: u32 nibble j = U[s][j]; width 2: u16 = G & 0xFFFF and
 *        width 1: u8 = G >> 16 of the 24-bit field G with bits 3j..3j+2 =
 *        L[s][j].
 *  Value row position p = 16g + 2m + h (g, m = 0..7, h = 0..1) holds channel
 *  16m + g + 8h.  int8 (T1): token r has a 128-byte row whose 16-byte chunk g
 *  (positions 16g..16g+15) is stored at chunk g ^ (r & 6).  int4 (T2, T3):
 *  tokens 2i and 2i+1 share a 128-byte block; its 16-byte chunk g ^ (2i & 6)
 *  holds chunk g (8 bytes, even position in the low nibble, two's
 *  complement) of token 2i, then that of token 2i+1.  Unused bits are 0.  Slots of tokens never written keep
 *  whatever the caller put there (zero the pools to compare pages byte for
 *  byte).  This grouping gives each decode lane one aligned block per token
 *  and each tensor-core thread its value fragments in contiguous,
 *  bank-conflict-free 16-byte loads.
 *
 *  Page table: int32 [H_kv][total_pages].  Bits 31..30 = tier (0 drop, 1..3),
 *  bits 29..0 = page index inside that tier's pool.  Sequence b owns logical
 *  pages page_offsets[b] .. page_offsets[b+1]-1 (for every kv head); token
 *  position p lives in logical page p / 16, slot p % 16.  Query head h reads
 *  kv head h / (H_q / H_kv).
 */
#ifndef SPHKV_H
#define SPHKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int sphkv_status;
#define SPHKV_OK 0
#define SPHKV_ERR_ARG 1      /* null/misaligned pointer, bad size or shape */
#define SPHKV_ERR_RANGE 2    /* radius or value scale overflows fp16; context > capacity */
#define SPHKV_ERR_BUDGET 3   /* RDR: the forced pages alone exceed the budget */
#define SPHKV_ERR_DEVICE 4   /* a CUDA call or launch failed */
#define SPHKV_ERR_TIMEOUT 5  /* a bounded device-side wait ran out */
#define SPHKV_ERR_DATA 6     /* device saw a page id outside its pool, a bad tier or position */

#define SPHKV_PAGE_TOKENS 16
#define SPHKV_HEAD_DIM 128

#define SPHKV_DTYPE_F32 0
#define SPHKV_DTYPE_BF16 1

/* The paged cache.  A plain descriptor: every pointer is device memory owned
 * by the caller; the struct itself lives on the host and is read only during
 * the call that receives it. */
typedef struct sphkv_cache {
    int32_t B;                   /* sequences */
    int32_t H_kv;                /* kv heads */
    int64_t total_pages;         /* logical pages per kv head = page_offsets[B] */
    const int32_t* page_offsets; /* [B+1], non-decreasing, page_offsets[0] = 0 */
    const int32_t* seq_lens;     /* [B] tokens present; <= 16 * pages owned */
    int32_t* page_table;         /* [H_kv][total_pages] entries, format above */
    uint8_t* pool[3];            /* pools of T1, T2, T3 pages, 16-byte aligned */
    int64_t pool_pages[3];       /* capacity of each pool in pages */
} sphkv_cache;

/* Bytes of one page of tier t (1..3); 0 for anything else. */
int sphkv_page_bytes(int tier);

/* Message of the last host-side error of the calling thread ("" if none). */
const char* sphkv_last_error(void);

/*
 * sphkv_encode -- dense K/V rows -> tier pages (prefill and append).
 *   Spherical KV, Abstract (ADA: a key becomes a radius plus angle codes).
 *   K, V: [n_tok][H_kv][128], dtype SPHKV_DTYPE_BF16 or SPHKV_DTYPE_F32.
 *   tok_seq, tok_pos: [n_tok] int32, sequence and position of each row.
 *   For each row and kv head the page-table entry of (seq, pos / 16) picks the
 *   tier and pool page; the token is written to slot pos % 16 of that page.
 *   Dropped pages are skipped.  Append is the same call with one row per
 *   sequence.  Codes are computed in fp64 with no fused multiply-add, so they
 *   match a plain fp64 reference bit for bit (short of libm atan2 differing in
 *   the last ulp at an exact rounding boundary).
 *   status_dev gets SPHKV_ERR_DATA for an out-of-range seq/pos/pool page
 *   (the row is skipped) and SPHKV_ERR_RANGE for an fp16 overflow.
 */
sphkv_status sphkv_encode(const sphkv_cache* cache, const void* K, const void* V, int dtype,
                          const int32_t* tok_seq, const int32_t* tok_pos, int64_t n_tok,
                          int32_t* status_dev, void* stream);

/*
 * sphkv_rdr_workspace_bytes / sphkv_rdr_assign -- rate-distortion retention.
 *   Spherical KV, Abstract (RDR: keep/drop and precision tiers chosen under
 *   a fixed byte budget as a rate-distortion trade-off); the Lagrangian form
 *   is this library's reading.  Units are (kv head g, sequence b, page p) for
 *   p < ceil(seq_len[b] / 16).  Page utility U = sum of `utility` over the
 *   page's present tokens, summed in slot order in fp64.  Rate R = page bytes
 *   of the tier (drop 0), distortion D = U * eps[tier].  The first n_sink and
 *   last n_recent pages of each sequence are forced to T1 and count against the
 *   budget.  Every other unit takes argmin_t U*eps[t] + lambda*R[t] (fp64, no
 *   FMA, ties to the higher precision); lambda starts at 1, doubles until the
 *   bytes fit (at most 2000 times), then 100 bisection steps keep the feasible
 *   end.  The whole search runs on the device in one cooperative kernel.
 *   utility: [H_kv][total_pages * 16] float (slot s of logical page i at
 *            i * 16 + s).
 *   eps: host [4] distortion per unit utility of T1, T2, T3, drop.
 *   tiers_out: [H_kv][total_pages] uint8, written 1..3 (0 = drop) for pages
 *            that hold tokens; other entries untouched.
 *   lambda_out: device double; bytes_out: device int64 (total bytes chosen).
 *   status_dev gets SPHKV_ERR_BUDGET when the forced pages exceed the budget
 *   (tiers_out is then left untouched).
 *   workspace: device, at least sphkv_rdr_workspace_bytes(...) bytes.
 */
size_t sphkv_rdr_workspace_bytes(int32_t B, int32_t H_kv, int64_t total_pages);
sphkv_status sphkv_rdr_assign(const sphkv_cache* cache, const float* utility, const double* eps,
                              int64_t budget_bytes, int32_t n_sink, int32_t n_recent,
                              uint8_t* tiers_out, double* lambda_out, int64_t* bytes_out,
                              void* workspace, size_t ws_bytes, int32_t* status_dev,
                              void* stream);

/*
 * sphkv_rdr_rerun -- RDR again on a cache whose pages already hold codes, as
 *   the context grows.  Spherical KV, AI Summary (retention allocates
 *   precision and storage dynamically by estimated future utility).  Reading:
 *   a page's codes can only be made coarser without the dense key, so each
 *   unit chooses among its current tier and the coarser ones (drop included);
 *   forced units (first n_sink, last n_recent pages) keep the finest tier they
 *   are allowed (T1 if they are T1, else their current tier).  Otherwise
 *   exactly sphkv_rdr_assign, with the same workspace.
 *   tiers_io: [H_kv][total_pages] uint8, the current tiers on entry (every
 *   page that holds tokens), the new ones on return.  Apply the result with
 *   sphkv_build_page_table into new pools and sphkv_migrate.
 */
sphkv_status sphkv_rdr_rerun(const sphkv_cache* cache, const float* utility, const double* eps,
                             int64_t budget_bytes, int32_t n_sink, int32_t n_recent, uint8_t* tiers_io,
                             double* lambda_out, int64_t* bytes_out, void* workspace, size_t ws_bytes,
                             int32_t* status_dev, void* stream);

/*
 * sphkv_migrate -- rewrite a cache's tokens into new pools after its tiers
 *   changed (sphkv_rdr_rerun), transcoding from the stored codes alone; this
 *   also compacts the pools to the new tier counts.  Reading (the pages give
 *   no rule): each angle goes to the nearest point of the coarser grid,
 *   computed exactly on the code integers with ties to even (leaf c ->
 *   rne(c 2^b' / 2^b) mod 2^b', upper c -> rne(c (2^b' - 1) / (2^b - 1)));
 *   the radius and its drop flag are kept; values are decoded (code x scale,
 *   exact in fp64) and quantised again with the encoder's rule (new scale
 *   fp16(max|v| / Q), codes clamp(rint(v / scale), -Q, Q)).  A token whose
 *   tier does not change moves unchanged.  Bit-exact with a plain reference.
 *   from: the old cache; to: the same sequences (B, H_kv, total_pages,
 *   page_offsets, seq_lens) with the new page table and new pools, which the
 *   caller zeroes first.  Every present token of every page `to` keeps is
 *   written; pages `to` drops are skipped.  status_dev gets SPHKV_ERR_DATA
 *   for a page that `to` makes finer than `from`, or keeps although `from`
 *   dropped it (codes cannot be recovered), or a pool page out of range.
 */
sphkv_status sphkv_migrate(const sphkv_cache* from, const sphkv_cache* to, int32_t* status_dev, void* stream);

/*
 * sphkv_build_page_table -- tiers -> page-table entries.
 *   Spherical KV, Abstract (each page holds one tier, with little metadata
 *   per page).  tiers: [n_entries] uint8 (0 drop, 1..3) in table order; the
 *   k-th entry of tier t (in table order) gets pool page perm_t[k], or k when
 *   perm_t is NULL.  table: [n_entries] int32 out.  counts_out: device int64[3]
 *   pages used per tier (may be NULL).  One kernel, a block-wide scan.
 *   status_dev gets SPHKV_ERR_DATA if a tier value is above 3.
 */
sphkv_status sphkv_build_page_table(const uint8_t* tiers, int64_t n_entries, const int32_t* perm1,
                                    const int32_t* perm2, const int32_t* perm3, int32_t* table,
                                    int64_t* counts_out, int32_t* status_dev, void* stream);

/*
 * sphkv_decode_workspace_bytes / sphkv_decode_attention -- ADA decode.
 *   Spherical KV, Abstract (logits come from the codes themselves, no dense
 *   key is rebuilt, over paged block-local storage).  One decode query per
 *   sequence.
 *   q: [B][H_q][128] fp32.  out: [B][H_q][128] fp32 = softmax-weighted sum of
 *   the dequantised values of the kept tokens (t < seq_len, page not dropped);
 *   lse: [B][H_q] fp32, natural-log log-sum-exp of the logits (scale 1/sqrt(d)
 *   included).  A head with no kept token gets out = 0, lse = -inf.
 *   H_q / H_kv must be 4.  Long contexts are split across SMs and the partial
 *   (max, sum, out) triples merged with a log-sum-exp combine; the split
 *   depends only on the shapes and the SM count, so results are reproducible
 *   bit for bit and independent of the pool page ids.
 *   workspace: device, 256-byte aligned, at least
 *   sphkv_decode_workspace_bytes(B, H_q, H_kv, total_pages, n_sm) bytes, where
 *   n_sm = 0 means the current device's SM count.
 */
size_t sphkv_decode_workspace_bytes(int32_t B, int32_t H_q, int32_t H_kv, int64_t total_pages,
                                    int32_t n_sm);
sphkv_status sphkv_decode_attention(const sphkv_cache* cache, int32_t H_q, const float* q,
                                    float* out, float* lse, void* workspace, size_t ws_bytes,
                                    int32_t* status_dev, void* stream);

/*
 * sphkv_decode_attention_noalloc -- sphkv_decode_attention without a caller
 *   workspace.  The paper has no counterpart: this entry point exists for
 *   callers that cannot allocate device memory, such as an engine that owns
 *   every byte of device memory and forbids allocation after start-up, or a
 *   latency-critical loop where cudaMalloc and the synchronisation it can
 *   imply are not acceptable.  It allocates nothing: the decode scratch (unit
 *   page offsets and split-KV partials) lives in a 4 MiB static device array
 *   inside the library, which every GPU that loads the library holds until
 *   the process exits.  Arguments, results and errors are those of
 *   sphkv_decode_attention; q, out and lse are still the caller's.
 *   - A cache whose scratch need (sphkv_decode_workspace_bytes with n_sm = 0)
 *     exceeds 4 MiB is rejected with SPHKV_ERR_ARG and a message naming both
 *     sizes; nothing is launched.
 *   - Every call looks up the array's device address with the caller's device
 *     current (no allocation; the address stays right across a device reset).
 *     The first call on a device also loads the library's kernels there: make
 *     that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (every value the kernels read is written earlier in the same
 *     call, so nothing needs clearing).  Calls whose work overlaps on the GPU,
 *     e.g. on two streams, race on it: serialise them.
 */
sphkv_status sphkv_decode_attention_noalloc(const sphkv_cache* cache, int32_t H_q, const float* q,
                                            float* out, float* lse, int32_t* status_dev, void* stream);

/*
 * sphkv_decode_mq_workspace_bytes / sphkv_decode_attention_mq -- ADA decode
 *   for n_q query tokens per sequence at once (speculative or chunked decode).
 *   Spherical KV, Abstract (the decode path is meant to fuse with the
 *   surrounding decode work); the multi-token form is this library's reading:
 *   query token i (0 <= i < n_q) of sequence b is causal, it sees the first
 *   seq_len[b] - (n_q - 1 - i) tokens (the last query token sees them all;
 *   the cache already holds the tokens the earlier queries precede), and
 *   otherwise attends exactly as in sphkv_decode_attention.
 *   q: [B][n_q][H_q][128] fp32, out: [B][n_q][H_q][128] fp32, lse:
 *   [B][n_q][H_q] fp32.  A query that sees no kept token gets out = 0,
 *   lse = -inf.  Query tokens are taken two at a time: one pass over the pages
 *   serves both (8 query heads per kv head on the tensor-core tile); an odd
 *   last token runs alone.  Pages are therefore read ceil(n_q / 2) times.
 *   1 <= n_q <= 1024, H_q / H_kv must be 4.  workspace: device, 256-byte
 *   aligned, at least sphkv_decode_mq_workspace_bytes(B, H_q, H_kv,
 *   total_pages, n_sm) bytes (n_sm = 0: the current device's SM count); the
 *   launches of one call reuse it in stream order.  Errors as
 *   sphkv_decode_attention, plus SPHKV_ERR_ARG for n_q out of range.
 */
size_t sphkv_decode_mq_workspace_bytes(int32_t B, int32_t H_q, int32_t H_kv, int64_t total_pages,
                                       int32_t n_sm);
sphkv_status sphkv_decode_attention_mq(const sphkv_cache* cache, int32_t n_q, int32_t H_q, const float* q,
                                       float* out, float* lse, void* workspace, size_t ws_bytes,
                                       int32_t* status_dev, void* stream);

/*
 * sphkv_set_keep -- per-token keep/drop inside kept pages.
 *   Spherical KV, Abstract (RDR makes keep/drop decisions per token and
 *   head).  Format: the sign bit of a token's stored radius is its drop flag
 *   (a radius fp16(|k|) is never negative, so the bit is otherwise always 0):
 *   decode skips a dropped token exactly as if it were absent (a head whose
 *   tokens are all dropped gets out = 0, lse = -inf).  Page sizes do not
 *   change; sphkv_encode writes tokens as kept.
 *   keep: [H_kv][total_pages * 16] uint8, the layout of sphkv_rdr_assign's
 *   utility (slot s of logical page i at i * 16 + s); nonzero = keep.  For
 *   every present token (position < seq_len) of every page that is not
 *   dropped, the flag is cleared (keep) or set (drop); other bytes are not
 *   touched.  status_dev gets SPHKV_ERR_DATA for a pool page out of range.
 */
sphkv_status sphkv_set_keep(const sphkv_cache* cache, const uint8_t* keep, int32_t* status_dev, void* stream);

/*
 * sphkv_merge_partials -- combine decode results computed over disjoint parts
 *   of the same sequences (split-KV across GPUs: each GPU decodes its own
 *   contiguous range of a long stream's pages, then the parts are gathered).
 *   Spherical KV, Abstract (long-context inference); the log-sum-exp combine
 *   is the one sphkv_decode_attention uses for its own split pieces.  With
 *   M = max_r lse_r and w_r = exp(lse_r - M):
 *     out = sum_r w_r out_r / sum_r w_r,   lse = M + ln sum_r w_r.
 *   A part with lse = -inf (no kept token) contributes nothing; a row whose
 *   parts are all empty gets out = 0, lse = -inf.
 *   out_parts: [n_parts][n_rows][128] fp32, lse_parts: [n_parts][n_rows] fp32
 *   (e.g. n_rows = B * H_q for single-token decode), out: [n_rows][128],
 *   lse: [n_rows].  1 <= n_parts <= 4096.  One kernel launch on `stream`.
 */
sphkv_status sphkv_merge_partials(const float* out_parts, const float* lse_parts, int32_t n_parts,
                                  int64_t n_rows, float* out, float* lse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPHKV_H */
