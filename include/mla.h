/*
 * mla.h - C ABI of the B200 (sm_100a) weight-absorbed MLA decode library (libmla.so).
 *
 * The library computes one decode step of Multi-head Latent Attention over a paged
 * cache that holds, per token, only the rank-r latent c_kv and the rotated RoPE key
 * of every key group. The four compute calls follow the absorbed order of the
 * DeepSeek-V2 MLA page (dtcms.com, "Matrix absorption" section):
 *
 *   mla_cache_append  write c_kv and RoPE(k_r) of new tokens into the paged cache
 *   mla_absorb_q      q_c = einsum('hdc,bhqd->bhqc', W_UK, q_nope), RoPE(q_pe) -> q_ext
 *   mla_decode_attn   scores = q_pe.k_pe + q_c.c_kv, scaled, softmaxed;
 *                     o_ = einsum('bhql,blc->bhqc', attn, c_kv)   (einsum 4) and lse
 *   mla_out_up        o = einsum('bhqc,hdc->bhqd', o_, W_UV) (+ bias)  (einsum 5)
 *   mla_decode_step   the four above in one call (the append folded into the absorption)
 *
 * Conventions shared by every call
 *   - Every data pointer is DEVICE memory owned by the caller; the library allocates
 *     nothing and keeps no state between calls that a result depends on, so concurrent
 *     calls on different streams are safe as long as their output buffers differ. Two
 *     exceptions: mla_decode_attn_noalloc's fixed scratch array (one call at a time, see
 *     there), and a mutex-guarded, per-device memo of a hardware property (how many
 *     two-CTA clusters of the decode fit on the device at once, which is constant for a
 *     device and shared-memory size).
 *   - bf16 tensors are passed as void* (uint16 storage), contiguous, row-major, in the
 *     shapes given below; fp32 and int32 tensors likewise.
 *   - Calls are asynchronous on `stream` (a cudaStream_t / CUstream; NULL = the legacy
 *     default stream). The returned status covers host-side argument validation and
 *     launch errors only; nothing is launched when validation fails.
 *   - Faults the device detects (a page id outside [0, num_pages), a context length
 *     outside the bounds the call was planned for, a pipeline wait that ran out) set
 *     bits in a caller-owned int32 "device error word"; read it with
 *     mla_get_device_status. Kernels only OR bits into the word, never clear it.
 *
 * Shapes use: B batch, q query tokens per sequence, H query heads, G key groups
 * (1 = one k_pe shared by all heads), r = kv_lora_rank, d_n = qk_nope_dim,
 * d_r = rope_dim per group, d_v = v_head_dim, ps = page_size, D = r + G*d_r the
 * cache row width. Head h uses key group g(h) = h / (H / G).
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, inconsistent dims          */
  MLA_ERR_UNSUPPORTED = 2,    /* valid but not implemented shape (never a fallback) */
  MLA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than required         */
  MLA_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed                   */
  MLA_ERR_DEVICE_BOUNDS = 5,  /* device saw an out-of-range page id or length        */
  MLA_ERR_DEVICE_TIMEOUT = 6  /* a device pipeline wait exceeded its limit           */
} mla_status;

/* Bits a kernel ORs into the device error word. */
#define MLA_DEVERR_BOUNDS (1 << 0)
#define MLA_DEVERR_TIMEOUT (1 << 1)

typedef struct mla_dims {
  int32_t num_heads;     /* H                                                    */
  int32_t num_kv_groups; /* G, divides H                                         */
  int32_t kv_lora_rank;  /* r, multiple of 8                                     */
  int32_t qk_nope_dim;   /* d_n, multiple of 8                                   */
  int32_t rope_dim;      /* d_r per group, even (0 allowed)                      */
  int32_t v_head_dim;    /* d_v, multiple of 8                                   */
  int32_t page_size;     /* tokens per cache page                                */
  float softmax_scale;   /* multiplies q.k before the softmax                    */
} mla_dims;

/* Cache row width D = r + G*d_r, or -1 when `dims` is null or inconsistent. */
int32_t mla_row_width(const mla_dims* dims);

/* Human-readable name of a status code (static string). */
const char* mla_status_string(mla_status status);

/*
 * mla_cache_append - write n_new tokens per sequence into the paged latent cache.
 *
 * Defined by the MLAfication data flow (wzjinhao.cn page: the KV cache stores only
 * c_kv plus the low-dimensional rotary key) and the row layout
 * torch.split(compressed_kv, [kv_lora_rank, qk_rope_head_dim]) of the DeepSeek-V2 page;
 * the cached key is post-RoPE, as only q_pe is rotated at attention time there.
 *
 *   c_kv        bf16 [B, n_new, r]          latent of each new token (copied bit-exactly)
 *   k_r         bf16 [B, n_new, G, d_r]     unrotated rotary key of each new token
 *   rope_cos/sin fp32 [B, n_new, G, d_r/2]  cos/sin of each pair's angle at the token's
 *                                           position; pair j is (x_j, x_{j+d_r/2})
 *   block_table int32 [B, max_pages_per_seq] physical page of each logical page
 *   start_pos   int32 [B]                   position of the first new token
 *   cache       bf16 [num_pages, ps, D]     updated in place
 *   dev_error   int32 device error word (may be NULL: faults are then only skipped)
 *
 * Token t of sequence b at position p = start_pos[b] + t goes to page
 * block_table[b][p / ps], row p % ps: cache[.., 0:r] = c_kv and, for each group g,
 * cache[.., r + g*d_r ...] = bf16_rne(x0*c - x1*s | x1*c + x0*s) with every product
 * and sum rounded to fp32 separately. A page id outside [0, num_pages) or a logical
 * page outside the table sets MLA_DEVERR_BOUNDS and that token is skipped.
 */
mla_status mla_cache_append(const mla_dims* dims, const void* c_kv, const void* k_r,
                            const float* rope_cos, const float* rope_sin,
                            const int32_t* block_table, int32_t max_pages_per_seq,
                            const int32_t* start_pos, int32_t batch, int32_t n_new,
                            void* cache, int64_t num_pages, int32_t* dev_error,
                            void* stream);

/*
 * mla_down_kv_append - the KV down-projection of new tokens, written straight into the
 * paged cache: one tcgen05 GEMM whose epilogue is mla_cache_append.
 *
 * The MLAfication page (wzjinhao.cn) sends the hidden state X through down_kv to the
 * latent c_kv (all the cache keeps of K/V) and through k_r_proj to the rotary key; the
 * DeepSeek-V2 page does both with kv_a_proj_with_mqa, eq. (41), split into
 * [kv_lora_rank, qk_rope_head_dim].
 *
 *   hidden      bf16 [B, n_new, hidden_dim]   hidden_dim a multiple of 8
 *   w_dkv       bf16 [D, hidden_dim]          rows 0..r-1: down_kv; rows r + g*d_r + j:
 *                                             group g's k_r_proj (no bias)
 *   rope_cos/sin, block_table, start_pos, cache, num_pages, dev_error: as mla_cache_append
 *   kv_out      bf16 [B, n_new, D] or NULL    if given, also receives the GEMM's bf16
 *                                             output [c_kv ; k_r] before the rotation
 *
 * For each token: [c_kv ; k_r] = bf16_rne(fp32 sum over hidden of w_dkv * x), then exactly
 * what mla_cache_append writes for that c_kv and k_r (the same cache bytes). The sum over
 * the model width is split across the CTAs of a cluster and added in a fixed order, so
 * every call gives the same bits. Needs no workspace. Requires G*d_r <= 128
 * (MLA_ERR_UNSUPPORTED otherwise). Bounds faults as mla_cache_append.
 */
mla_status mla_down_kv_append(const mla_dims* dims, const void* hidden, int32_t hidden_dim,
                              const void* w_dkv, const float* rope_cos, const float* rope_sin,
                              const int32_t* block_table, int32_t max_pages_per_seq,
                              const int32_t* start_pos, int32_t batch, int32_t n_new,
                              void* cache, int64_t num_pages, int32_t* dev_error, void* kv_out,
                              void* stream);

/*
 * mla_absorb_q - fold W_UK into the query and rotate its RoPE part.
 *
 * The "W^{UK} is absorbed by q_nope" step of the DeepSeek-V2 page:
 * q_c = einsum('hdc,bhqd->bhqc', q_absorb, q_nope), and q_pe = apply_rotary_pos_emb
 * at the query positions.
 *
 *   q_nope      bf16 [B, q, H, d_n]
 *   q_pe        bf16 [B, q, H, d_r]         unrotated
 *   rope_cos/sin fp32 [B, q, G, d_r/2]      angles at each query row's position
 *   w_uk        bf16, head h at w_uk + h*w_uk_head_stride (elements), each [d_n, r]
 *               row-major; w_uk_head_stride >= d_n*r, multiple of 8 (a packed
 *               kv_b_proj view [H, d_n + d_v, r] passes stride (d_n + d_v)*r)
 *   q_ext       bf16 [B, q, H, D] output:   [0:r) = q_c (fp32 accumulate, bf16 round),
 *               [r + g(h)*d_r, +d_r) = RoPE(q_pe) (fp32, bf16 round), other groups 0
 */
mla_status mla_absorb_q(const mla_dims* dims, const void* q_nope, const void* q_pe,
                        const float* rope_cos, const float* rope_sin, const void* w_uk,
                        int64_t w_uk_head_stride, int32_t batch, int32_t q_len, void* q_ext,
                        void* stream);

/*
 * mla_out_proj - einsums (5) and (6) of the DeepSeek-V2 page's "Matrix absorption" section
 * in one kernel: the value up-projection o = einsum('bhqc,hdc->bhqd', o_, W_UV) (+ up_v bias)
 * followed by the output projection u = einsum('hdD,bhqd->bqD', W_o, o) (+ bias), the
 * latter being the page's o_proj of size [num_heads * v_head_dim, hidden_size].
 *
 *   o_latent  bf16 [rows, H, r]             rows = B*q (mla_decode_attn's o_latent)
 *   w_uv, w_uv_head_stride, bias_v          as mla_out_up (bias_v [H, d_v] or NULL)
 *   w_o       bf16 [hidden, H*d_v]          row k holds W_o[h, d, k] at column h*d_v + d
 *                                           (a torch.nn.Linear(H*d_v, hidden) weight)
 *   bias_o    bf16 [hidden] or NULL
 *   workspace >= mla_out_proj_workspace_size(dims, hidden, rows) bytes, 256-byte aligned,
 *             zeroed once after allocation; the call leaves its counters zero again, so
 *             the workspace serves later calls on the same stream (not concurrent ones).
 *             Its first int32 is a device error word (MLA_DEVERR_TIMEOUT if a wait ran out).
 *   o         bf16 [rows, H, d_v] output (the up-projected values, also the input of (6))
 *   u         bf16 [rows, hidden] output (fp32 accumulate; stage (6) adds its K splits in
 *             a fixed order, so the result is deterministic)
 * Requires d_v % 64 == 0 and hidden % 8 == 0 (MLA_ERR_UNSUPPORTED / MLA_ERR_INVALID_ARG).
 * The kernel is a cooperative launch (all its CTAs resident at once, one per SM); it fails
 * with MLA_ERR_CUDA if the device cannot hold them.
 */
size_t mla_out_proj_workspace_size(const mla_dims* dims, int32_t hidden, int32_t rows);
mla_status mla_out_proj(const mla_dims* dims, const void* o_latent, const void* w_uv,
                        int64_t w_uv_head_stride, const void* bias_v, const void* w_o,
                        const void* bias_o, int32_t hidden, int32_t rows, void* workspace,
                        size_t workspace_bytes, void* o, void* u, void* stream);

/*
 * Bytes of workspace mla_decode_attn needs for this problem (0 on invalid input).
 * num_splits: 0 lets the library size the grid (one CTA per SM); n > 0 asks for n
 * equal work ranges per (sequence, block of query rows) on average. The workspace holds
 * the device error word (int32 at offset 0; zero it once after allocating), the
 * schedule and the partial results of sequences cut between CTAs. A workspace can be
 * reused by later calls on the same stream, not by calls running concurrently.
 */
size_t mla_decode_workspace_size(const mla_dims* dims, int32_t batch, int32_t q_len,
                                 int32_t max_seq_len, int32_t num_splits);

/*
 * mla_decode_attn - paged, split-KV absorbed attention over the latent cache.
 *
 * For sequence b with context length L = seq_lens[b] (after the append) and query row
 * i at position L - q + i, every head h scores each visible token l (l <= L - q + i
 * when causal != 0, else every l < L):
 *     s = softmax_scale * (q_ext[b,i,h,:] . cache_row(b, l))
 * (the q_pe.k_pe + q_c.c_kv of the DeepSeek-V2 page, since q_ext zero-pads the other
 * groups' rotary slots), p = softmax over l, and writes
 *     o_latent[b,i,h,:] = sum_l p * c_kv[l]      (einsum 4, bf16)
 *     lse[b,i,h]        = ln sum_l exp(s)        (fp32)
 * The cached pages of all sequences are cut into equal ranges, one per CTA, so ragged
 * lengths balance; a sequence cut between CTAs is merged with the log-sum-exp identity
 * by a second, small kernel launched right after.
 *
 *   q_ext       bf16 [B, q, H, D]   from mla_absorb_q
 *   cache       bf16 [num_pages, ps, D]
 *   block_table int32 [B, max_pages_per_seq]
 *   seq_lens    int32 [B], each in [q, max_seq_len] and <= max_pages_per_seq*ps
 *   max_seq_len host-side upper bound of seq_lens, used to plan the splits
 *   o_latent    bf16 [B, q, H, r] output; lse fp32 [B, q, H] output
 *   workspace   >= mla_decode_workspace_size(...) bytes, 256-byte aligned
 * Supported: ps == 64, H*q rows split in groups of <= 64 per CTA, r <= 512,
 * D <= 640. Others return MLA_ERR_UNSUPPORTED.
 */
mla_status mla_decode_attn(const mla_dims* dims, const void* q_ext, const void* cache,
                           int64_t num_pages, const int32_t* block_table,
                           int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                           int32_t q_len, int32_t max_seq_len, int32_t causal,
                           int32_t num_splits, void* workspace, size_t workspace_bytes,
                           void* o_latent, float* lse, void* stream);

/*
 * mla_decode_step - one whole decode step in one call: mla_cache_append, mla_absorb_q,
 * mla_decode_attn and mla_out_up on the same arguments, in that order (the absorbed
 * order of the DeepSeek-V2 page's "Matrix absorption" section, einsums (4) and (5)).
 * Every output is the one the four calls would produce, bit for bit. The append is
 * folded into the absorption kernel (its rows are written while the first weight tiles
 * arrive), so the step launches three kernels (four when the decode plan cuts sequences
 * between CTAs and runs its merge).
 *
 *   c_kv_new, k_r_new, rope_cos_new, rope_sin_new, start_pos, n_new
 *                              as mla_cache_append's c_kv, k_r, rope_cos, rope_sin,
 *                              start_pos, n_new (n_new = 0: nothing appended)
 *   q_nope, q_pe, rope_cos_q, rope_sin_q, w_uk, w_uk_head_stride
 *                              as mla_absorb_q
 *   w_uv, w_uv_head_stride, bias_v
 *                              as mla_out_up
 *   cache ... num_splits, workspace, workspace_bytes, o_latent, lse
 *                              as mla_decode_attn
 *   q_ext                      bf16 [B, q, H, D] scratch for the absorbed query (written)
 *   o                          bf16 [B, q, H, d_v] output
 * The append reports bounds faults into the workspace's device error word (its first
 * int32), like the decode. Every argument is validated before anything is launched;
 * the statuses are those of the four calls.
 */
mla_status mla_decode_step(const mla_dims* dims, const void* c_kv_new, const void* k_r_new,
                           const float* rope_cos_new, const float* rope_sin_new,
                           const int32_t* start_pos, int32_t n_new, const void* q_nope,
                           const void* q_pe, const float* rope_cos_q, const float* rope_sin_q,
                           const void* w_uk, int64_t w_uk_head_stride, const void* w_uv,
                           int64_t w_uv_head_stride, const void* bias_v, void* cache,
                           int64_t num_pages, const int32_t* block_table,
                           int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                           int32_t q_len, int32_t max_seq_len, int32_t causal,
                           int32_t num_splits, void* q_ext, void* workspace,
                           size_t workspace_bytes, void* o_latent, float* lse, void* o,
                           void* stream);

/*
 * mla_out_up - apply the value up-projection to the attention output (einsum 5 of the
 * DeepSeek-V2 page, o = einsum('bhqc,hdc->bhqd', o_, W_UV)), plus the optional up_v
 * bias of the MLAfied checkpoints (wzjinhao.cn page). Exact under absorption because
 * softmax weights sum to one.
 *
 *   o_latent  bf16 [rows, H, r]   rows = B*q
 *   w_uv      bf16, head h at w_uv + h*w_uv_head_stride (elements), each [d_v, r]
 *   bias      bf16 [H, d_v] or NULL
 *   o         bf16 [rows, H, d_v] output (fp32 accumulate)
 */
mla_status mla_out_up(const mla_dims* dims, const void* o_latent, const void* w_uv,
                      int64_t w_uv_head_stride, const void* bias, int32_t rows, void* o,
                      void* stream);

/*
 * The single-latent K = V form (nanowhale-100m page, cnnetsun.cn: "single KV head, many
 * query heads", "applying RoPE" and "efficient attention", where
 * scaled_dot_product_attention(q, kv_expanded, kv_expanded) uses one head_dim vector per
 * token as both key and value, RoPE on its last d_r dims, and the output's rotary dims are
 * rotated back afterwards).
 *
 * dims describe that form: num_kv_groups = 1, kv_lora_rank = r = the unrotated width,
 * qk_nope_dim = r, rope_dim = d_r > 0, v_head_dim = r + d_r = D (the head_dim). The cache is
 * the ordinary latent cache written by mla_cache_append with these dims (row = [kv_nope |
 * RoPE(kv_pe)]). One decode step is then:
 *   mla_kv_shared_query   q_ext = [q[:r] ; R(pos) q[r:]]                (bf16 [B, q, H, D])
 *   mla_decode_attn       with the dims from mla_kv_shared_decode_dims (the whole row is
 *                         the "latent": rank D, no separate rotary slot), giving
 *                         o_latent = sum_l p_l row_l  [B, q, H, D] and lse
 *   mla_kv_shared_output  o = [o_latent[:r] ; R(-pos) o_latent[r:]]    (bf16 [B, q, H, D])
 * R(pos) rotates the pairs (x_j, x_{j+d_r/2}) by the caller's angles: rope_cos/sin fp32
 * [B, q, 1, d_r/2] at each query row's position (the same tables for both calls). The
 * rotation is fp32 with separately rounded products and sums, then bf16 round to nearest
 * even. A model whose rotary embedding pairs adjacent dims (complex form) permutes its
 * rotary dims once to this half-split layout; attention and the inverse rotation commute
 * with that permutation.
 *
 * mla_kv_shared_decode_dims: writes the decode view of `dims` ({H, 1, D, D, 0, D, ps,
 * scale}) to `decode_dims`; MLA_ERR_INVALID_ARG if `dims` is not a K = V layout.
 * mla_kv_shared_query / _output: q / o_latent and q_ext / o are [B, q, H, D] bf16, 16-byte
 * aligned; in place allowed (in == out). MLA_ERR_INVALID_ARG on a non-K = V layout, a null
 * or misaligned pointer, batch < 0 or q_len <= 0; batch == 0 launches nothing.
 */
mla_status mla_kv_shared_decode_dims(const mla_dims* dims, mla_dims* decode_dims);
mla_status mla_kv_shared_query(const mla_dims* dims, const void* q, const float* rope_cos,
                               const float* rope_sin, int32_t batch, int32_t q_len, void* q_ext,
                               void* stream);
mla_status mla_kv_shared_output(const mla_dims* dims, const void* o_latent,
                                const float* rope_cos, const float* rope_sin, int32_t batch,
                                int32_t q_len, void* o, void* stream);

/*
 * mla_decode_attn_noalloc - mla_decode_attn for callers that cannot allocate device memory.
 *
 * The pages have no counterpart for this call; it exists for deployment. Code that runs
 * where cudaMalloc is not allowed (inside an allocator or memory-pool hook that must not
 * re-enter the allocator, or a runtime that fixes its device-memory budget at start-up)
 * cannot provide mla_decode_attn's workspace. This variant computes the same o_latent and
 * lse with the workspace replaced by a fixed scratch array of MLA_NOALLOC_SCRATCH_BYTES
 * that the library keeps in its own device memory; every GPU that loads the library holds
 * that array until the process exits. It never calls cudaMalloc or cudaFree.
 *
 *   Arguments are those of mla_decode_attn without num_splits / workspace, plus
 *   dev_error: int32 device error word (required): bits the decode sets are ORed into it.
 *
 * - The first call on each device looks up the array's device address (a host-side
 *   runtime query, done once per device with that device current); make that first call
 *   before capturing the stream into a CUDA graph.
 * - All calls share the one array and it keeps the last call's contents; each call
 *   rewrites what it reads, so nothing has to be cleared between calls. Calls whose
 *   execution overlaps on the GPU (different streams, or different host threads without
 *   ordering) race on the array and must not be used.
 * - The call uses mla_decode_attn's automatic plan (num_splits = 0: at most one work range
 *   per SM), which needs the least workspace of all plans once there are more (sequence,
 *   block of query rows) units than SMs, and fits the array whenever there are fewer. A
 *   problem whose plan does not fit (millions of sequences, or many more row blocks than
 *   SMs) returns MLA_ERR_WORKSPACE and launches nothing.
 * - Validation is that of mla_decode_attn, done before anything else (batch == 0 included).
 */
#define MLA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
mla_status mla_decode_attn_noalloc(const mla_dims* dims, const void* q_ext, const void* cache,
                                   int64_t num_pages, const int32_t* block_table,
                                   int32_t max_pages_per_seq, const int32_t* seq_lens,
                                   int32_t batch, int32_t q_len, int32_t max_seq_len,
                                   int32_t causal, int32_t* dev_error, void* o_latent,
                                   float* lse, void* stream);

/*
 * Synchronise `stream`, read the device error word at `dev_error` and, if reset != 0,
 * clear it. Returns MLA_ERR_DEVICE_TIMEOUT, MLA_ERR_DEVICE_BOUNDS or MLA_OK (or
 * MLA_ERR_CUDA if the read fails). For mla_decode_attn the word is the first int32
 * of its workspace.
 */
mla_status mla_get_device_status(const int32_t* dev_error, int32_t reset, void* stream);

/*
 * Self-test of the device error path. Launches one CTA on `stream` that waits on an
 * mbarrier nothing arrives on, with the same bounded wait every kernel here uses (2 s).
 * The wait gives up, ORs MLA_DEVERR_TIMEOUT into the caller's int32 error word `dev_error`
 * and the kernel returns, so the context stays usable. Returns MLA_OK once launched
 * (MLA_ERR_INVALID_ARG for a null word, MLA_ERR_CUDA if the launch fails); read the word
 * with mla_get_device_status.
 */
mla_status mla_selftest_wait_timeout(int32_t* dev_error, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
