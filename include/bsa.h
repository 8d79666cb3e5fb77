/*
 * bsa.h -- C ABI of the B200 (sm_100a) BigBird block-sparse attention forward
 * and its gradients (bsa_backward).
 *
 * What the forward computes, for every batch element b, head h and
 * query token t of query block i = t / 64:
 *
 *     O[b,h,t,:] = softmax_{p in A(h,i)} ( q_t . k_p * scale ) . V[b,h,p,:]
 *     lse[b,h,t] = ln sum_{p in A(h,i)} exp( q_t . k_p * scale )
 *
 * where A(h,i) is the union of the key tokens of the key blocks listed in
 * row (h, i) of the layout, minus the keys the optional key-padding mask drops.
 * This is the masked attention Softmax(Q K^T / sqrt(d_k) (.) M) V of
 * "Adapt or Perish: 新手入门指南 – Adaptive Sparse Transformer 核心原理与实战"
 * (section on the sparse-attention formula), with (.) M read as restricting
 * the softmax to M -- the pages' own code fills the excluded scores with
 * -1e9 / -1e10 ("BERT 稀疏注意力机制入门指南", PyTorch 实现; "BERT多头注意力机制深度解析",
 * BlockSparseAttention).  A single softmax runs over the union of the three
 * BigBird patterns ("BigBird 稀疏注意力机制解析", 核心实现): global, sliding
 * window, random.  The mask is stored at 64x64 block granularity
 * ("Transformer计算效率优化：SQA稀疏注意力机制详解", 3.1 and 5 问题3).
 *
 * Conventions for every entry point:
 *   - Return value: BSA_OK (0) or a negative bsa_status.  No C++ exception
 *     crosses this boundary.  Arguments are validated before anything is
 *     launched; a failing call has no effect on the GPU.
 *   - "device" pointers are CUDA device pointers of the current device;
 *     "host" pointers are ordinary CPU memory.  The caller owns every buffer it
 *     passes in; the library owns the bsa_layout object and its device copies.
 *   - A stream argument is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  GPU work is enqueued asynchronously on it.
 *   - Thread safety: distinct layouts may be used concurrently; one layout may
 *     be shared by concurrent bsa_forward calls once uploaded (it is read-only
 *     then), each call with its own workspace.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = -1,     /* null pointer, bad size or range            */
  BSA_ERR_UNSUPPORTED = -2,     /* block not a multiple of 64, a head dim the
                                   call does not take, not an sm_100 device    */
  BSA_ERR_CUDA = -3,            /* a CUDA runtime/driver call failed           */
  BSA_ERR_LAYOUT_MISMATCH = -4, /* layout built for another H/L, or not uploaded
                                   to the current device                       */
  BSA_ERR_DEVICE_TIMEOUT = -5,  /* a bounded wait inside a kernel gave up      */
  BSA_ERR_OOM = -6,             /* host or device allocation failed            */
  BSA_ERR_WORKSPACE = -7,       /* workspace missing or too small              */
  BSA_ERR_STATIC_WORKSPACE = -8 /* problem needs more scratch than the library's
                                   built-in buffer (bsa_forward_static_ws)     */
} bsa_status;

/* Opaque, immutable after bsa_layout_build (bsa_layout_upload only adds
 * device copies).  Owned by the library; release with bsa_layout_free. */
typedef struct bsa_layout bsa_layout;

/*
 * bsa_layout_build -- host only, no GPU needed.
 *
 * Builds the BigBird block layout for H heads and sequence length L with
 * nb = L / block query/key blocks ("BigBird 稀疏注意力机制解析", 核心实现 and
 * 代码实现; window clipping from "BERT 稀疏注意力机制入门指南", PyTorch 实现):
 *   globals  G: if `globals` is non-NULL it holds n_global block indices (any
 *            order, duplicates allowed, each in [0, nb)); otherwise
 *            n_global == 0 -> {}, 1 -> {0}, else floor(k (nb-1)/(n_global-1)),
 *            k = 0..n_global-1, deduplicated (torch.linspace(...).long() of the
 *            page, in exact integers).
 *   row (h,i) for i in G: every block 0..nb-1.
 *   row (h,i) otherwise: window {j : |i-j| <= window, 0 <= j < nb} union G union
 *            R(h,i), where R(h,i) is min(n_random, m) distinct blocks drawn from
 *            the m blocks outside window and G by a partial Fisher-Yates
 *            shuffle (ascending candidate list; step t swaps entries t and
 *            t + u_t mod (m - t)) driven by the raw 64-bit outputs u_0, u_1, ...
 *            of Philox4x64-10 with key {seed, 0} and counter {0, i, h, 0},
 *            incremented (as a 256-bit little-endian integer) before each
 *            4-word block is produced.
 *   Rows are sorted ascending and duplicate-free; the layout is shared by all
 *   batch elements.  CSR rows are ordered head-major then query block.
 *
 * block must be a multiple of 64 (else BSA_ERR_UNSUPPORTED); L > 0 and
 * L % block == 0; H >= 1; window, n_global, n_random >= 0 (else
 * BSA_ERR_INVALID_ARG).  All of the above is in units of `block` (rows, window,
 * globals, the random draws' counter i).  The kernels run 64-key blocks: a
 * layout at block 64 m is expanded exactly, query block I's row becoming the
 * rows of its m 64-blocks, each listing the m 64-blocks of every key block in it
 * (the block size the pages leave to tuning, "Transformer计算效率优化：SQA稀疏注意力机制详解",
 * 5 问题3).  On success *out receives a new layout.
 */
int bsa_layout_build(int H, int L, int block, int window, int n_global, int n_random,
                     uint64_t seed, const int32_t* globals, bsa_layout** out);

/*
 * bsa_layout_build_tokens -- host only, no GPU needed.
 *
 * A BigBird layout whose window and global set are given in tokens, not whole
 * blocks ("BigBird 稀疏注意力机制解析", 核心实现 states the window in tokens).
 * Query token i of head h attends key token j when
 *     i in G  or  j in G  or  |i - j| <= window
 *     or  block(j) is a random block of block(i),
 * with blocks of 64 tokens and
 *   G        the global tokens: if `global_tokens` is non-NULL, its n_global
 *            token indices (each in [0, L), any order); otherwise n_global == 0
 *            -> {}, 1 -> {0}, else floor(k (L-1)/(n_global-1)), k = 0..n_global-1.
 *   random   for a block I holding no global token, min(n_random, m) blocks
 *            drawn as in bsa_layout_build (same Philox stream and shuffle) from
 *            the m blocks outside {J : |I - J| <= floor((window + 63) / 64)} and
 *            outside the blocks that hold a global token; none for the others.
 * The layout's block CSR (bsa_layout_csr) is the block layout those rules
 * touch: bsa_layout_build at block 64 with window floor((window + 63) / 64)
 * blocks and the blocks holding a global token as its globals.  The forward
 * applies the token rule inside the block pairs that need it (a per-row mask of
 * the pair's 64 keys), and so does bsa_backward (a mask of the key block's keys
 * per query row for dQ, of the query block's queries per key row for dK and dV).
 * L must be a positive multiple of 64; H >= 1;
 * window, n_global, n_random >= 0 (else BSA_ERR_INVALID_ARG).
 */
int bsa_layout_build_tokens(int H, int L, int window, int n_global, int n_random, uint64_t seed,
                            const int32_t* global_tokens, bsa_layout** out);

/*
 * bsa_layout_token_masks -- the token-level part of a layout from
 * bsa_layout_build_tokens: its window in tokens and a host view of L / 64
 * 64-bit words, bit c of word j set when token 64 j + c is global (valid until
 * bsa_layout_free).  Either output may be NULL.  BSA_ERR_UNSUPPORTED for a
 * block layout.
 */
int bsa_layout_token_masks(const bsa_layout* layout, int* window, const uint64_t** global_bits);

/*
 * bsa_layout_from_csr -- host only, no GPU needed.
 *
 * Builds a layout from a caller's block mask instead of the BigBird rule.
 * The pages keep the attention mask as a 0/1 matrix over 64x64 blocks
 * ("Transformer计算效率优化：SQA稀疏注意力机制详解", 3.1), and that is the CSR
 * form taken here.
 *   row_ptr  host, H*nb+1 int32 (nb = L / block): row (h, i), the key blocks
 *            query block i of head h attends, is col_idx[row_ptr[h*nb+i] ..
 *            row_ptr[h*nb+i+1]).  Rows are head-major.  row_ptr[0] must be 0
 *            and row_ptr must never decrease.
 *   col_idx  host, row_ptr[H*nb] int32 key block indices in [0, nb).  Within a
 *            row: any order, duplicates allowed; the layout keeps each row
 *            sorted and duplicate-free (bsa_layout_csr returns that form).
 *            May be NULL when row_ptr[H*nb] == 0.
 * A row may be empty: its query tokens get O = 0 and lse = -inf.  Rows may
 * differ between heads.  A query block that lists every key block in every
 * head is paired with other such blocks in the tile decomposition; such
 * blocks are what bsa_layout_globals returns for this layout.
 *
 * Rows that list every key block are how caller-chosen global query rows are
 * expressed, e.g. the top-k queries an SQA router picks for global attention
 * ("Transformer计算效率优化：SQA稀疏注意力机制详解", 2.1), the others keeping a
 * local window.
 *
 * block must be a multiple of 64 (else BSA_ERR_UNSUPPORTED); rows and
 * columns are in units of `block` and expanded to 64-key blocks as in
 * bsa_layout_build.  BSA_ERR_INVALID_ARG for H < 1, L < 1, L % block != 0, a
 * NULL row_ptr, a bad row_ptr or a column out of range.  The arrays are copied;
 * the caller keeps ownership.
 */
int bsa_layout_from_csr(int H, int L, int block, const int32_t* row_ptr, const int32_t* col_idx,
                        bsa_layout** out);

/*
 * bsa_layout_csr -- host views of the CSR in the layout's block units
 * (nb = L / block): row_ptr has H*nb+1 int32 entries, col_idx has nnz int32
 * entries (key block indices).  Any output pointer may be NULL.  The views stay
 * valid until bsa_layout_free.
 */
int bsa_layout_csr(const bsa_layout* layout, const int32_t** row_ptr,
                   const int32_t** col_idx, int64_t* nnz, int* nb, int* H);

/* bsa_layout_globals -- host view of the sorted global block list, in the
 * layout's block units. */
int bsa_layout_globals(const bsa_layout* layout, const int32_t** globals, int* n_global);

/*
 * bsa_layout_tiles -- host views of the 128-row tile decomposition the kernel
 * runs (two 64-row query blocks per tile over the union of their rows; block
 * indices here are always 64-key blocks).
 *   pair_q:   2*n_pairs int32, (first, second) query block; second = -1 when the
 *             tile holds a single block.  Global blocks pair with global blocks.
 *   pair_ptr: H*n_pairs+1 int32 offsets into pair_ent, head-major.
 *   pair_ent: key block | (membership << 24): bit 0 = in the first block's row,
 *             bit 1 = in the second's.  Per tile: the blocks in both rows, then
 *             the blocks in one row only, alternating first/second; each group
 *             ascending.
 * Any output may be NULL.
 */
/* Tiles whose union has more than BSA_SPLIT_THRESHOLD entries (global rows) are
 * cut into chunks of BSA_SPLIT_CHUNK entries; bsa_forward runs the chunks as
 * separate work items and merges their partial results in a second kernel. */
#define BSA_SPLIT_THRESHOLD 48
#define BSA_SPLIT_CHUNK 32
int bsa_layout_tiles(const bsa_layout* layout, const int32_t** pair_q, int* n_pairs,
                     const int32_t** pair_ptr, const uint32_t** pair_ent, int64_t* n_ent);

/*
 * bsa_layout_key_tiles -- host views of the key-major tiles the backward's dK/dV
 * kernel runs: the transposed layout (row (h, j) = the query blocks whose row
 * holds key block j, ascending) cut into 128-row tiles exactly as
 * bsa_layout_tiles describes for query rows.
 *   pair_k:   2*n_pairs int32, (first, second) key block; second = -1 for a
 *             single-block tile.  Key blocks that every query block attends in
 *             every head pair with each other.
 *   pair_ptr: H*n_pairs+1 int32 offsets into pair_ent, head-major.
 *   pair_ent: query block | (membership << 24): bit 0 = the query block attends
 *             the first key block, bit 1 = the second.  Order as in
 *             bsa_layout_tiles; a tile no query block attends holds one entry
 *             (block 0, no bits).
 * Any output may be NULL.
 */
int bsa_layout_key_tiles(const bsa_layout* layout, const int32_t** pair_k, int* n_pairs,
                         const int32_t** pair_ptr, const uint32_t** pair_ent, int64_t* n_ent);

/*
 * bsa_layout_upload -- copies the tile tables and work list to the CURRENT
 * device (cudaMemcpyAsync on `stream`, then a stream synchronize).  Must
 * precede bsa_forward on that device.  Calling it again re-uploads to the
 * then-current device.  Returns BSA_ERR_OOM / BSA_ERR_CUDA on failure.
 */
int bsa_layout_upload(bsa_layout* layout, void* stream);

/* bsa_layout_free -- releases host and device memory of the layout; NULL is a no-op. */
void bsa_layout_free(bsa_layout* layout);

/*
 * bsa_workspace_bytes -- device scratch bytes bsa_forward needs for batch size
 * B: the counters of the dynamic work schedule, the per-key-block padding bits
 * and the partial results of split rows (global rows whose key-block list is cut
 * into chunks that run as separate work items).  It needs no clearing: every
 * call first zeroes the 256 bytes of schedule counters it uses (one
 * cudaMemsetAsync on the call's stream) and writes every other byte before
 * reading it, so a workspace in any state -- fresh, reused, or left by a call
 * that ended in a device error -- can be passed.  Concurrent calls need
 * separate workspaces.
 */
int bsa_workspace_bytes(const bsa_layout* layout, int B, size_t* bytes);

/*
 * bsa_forward_workspace_bytes -- the same for head dim d (64 or 128; the partial
 * results of split rows hold d columns per row): bsa_workspace_bytes is this with
 * d = 64.  BSA_ERR_UNSUPPORTED for another d.
 */
int bsa_forward_workspace_bytes(const bsa_layout* layout, int B, int d, size_t* bytes);

/*
 * bsa_forward -- enqueues the block-sparse attention forward on `stream`.
 *   q, k, v   device, bf16, [B, H, L, d] contiguous, 16-byte aligned.
 *   d         64 or 128 (else BSA_ERR_UNSUPPORTED).  At d = 128 the kernel runs
 *             one pipeline per SM instead of two (its operands take twice the
 *             shared memory and TMEM).
 *   layout    built for this H and L and uploaded to the current device.
 *   key_mask  device uint8 [B, L] (1 = keep, 0 = drop the key), or NULL.
 *   scale     softmax scale applied to q.k; <= 0 selects 1/sqrt(d).
 *   out       device, bf16, [B, H, L, d] contiguous (round-to-nearest-even).
 *   lse       device, fp32, [B, H, L]: natural-log sum of exp of the scaled
 *             scores over the attended keys; -inf (with O = 0) for a row whose
 *             attended set is empty.
 *   workspace device, at least bsa_forward_workspace_bytes(layout, B, d) bytes
 *             (bsa_workspace_bytes at d = 64), 256-byte aligned, any contents
 *             (see above).
 * Enqueues on `stream` a 256-byte memset of the schedule counters and up to
 * three kernels: the key-padding bits (with a key mask), the forward, and the
 * merge of split rows (when the layout has any; it is launched as a
 * programmatic dependent of the forward, so its launch overlaps the forward's
 * end).  Key blocks whose 64 keys are all dropped by the key mask cost no
 * loads or MMAs.
 * Returns after enqueueing (no synchronisation, no allocation).  A device-side
 * timeout is reported later by bsa_sync_status.
 */
int bsa_forward(const void* q, const void* k, const void* v, int B, int H, int L, int d,
                const bsa_layout* layout, const uint8_t* key_mask, float scale,
                void* out, float* lse, void* workspace, size_t workspace_bytes,
                void* stream);

/*
 * bsa_forward_static_ws -- bsa_forward for callers that cannot allocate device
 * memory: code running where cudaMalloc is unavailable or forbidden, e.g. inside
 * a host runtime that owns every allocation, a plugin with no allocator hook, or
 * a path where an allocation would synchronise the device.  It allocates
 * nothing: the scratch (schedule counters, key-padding bits, split-row partials)
 * lives in one buffer of BSA_STATIC_WORKSPACE_BYTES (32 MiB) compiled into
 * the library, which every GPU that loads the library holds until process exit.
 * The pages define no such entry point; it has no counterpart there.
 *
 * Arguments and results are those of bsa_forward, minus the workspace.
 *   - Returns BSA_ERR_STATIC_WORKSPACE, before anything is enqueued, when
 *     bsa_workspace_bytes(layout, B) exceeds BSA_STATIC_WORKSPACE_BYTES.
 *   - The first call on a device looks up the buffer's device address for that
 *     device (cudaGetSymbolAddress, no allocation) and keeps it once the lookup
 *     succeeds (a failed lookup is retried by the next call); make that first
 *     call before any stream capture.  The kept address is not refreshed after
 *     cudaDeviceReset: do not reset a device between calls.
 *   - Every call clears the buffer's schedule counters with cudaMemsetAsync on
 *     `stream`, then enqueues the forward.  All calls on a device share the one
 *     buffer, which keeps the last call's contents: calls whose execution
 *     overlaps on the GPU (different streams, no ordering between them) race on
 *     it and give undefined results.  Serialise them.
 */
#define BSA_STATIC_WORKSPACE_BYTES (32u * 1024u * 1024u)
int bsa_forward_static_ws(const void* q, const void* k, const void* v, int B, int H, int L, int d,
                          const bsa_layout* layout, const uint8_t* key_mask, float scale,
                          void* out, float* lse, void* stream);

/*
 * bsa_backward_workspace_bytes -- device scratch bytes bsa_backward needs for
 * batch size B: key-padding bits, two fp32 values per query row (D and lse in
 * log2 units) and the fp32 partial sums of split tiles.  Unlike the forward's
 * workspace it needs no clearing: every byte is written before it is read.
 */
int bsa_backward_workspace_bytes(const bsa_layout* layout, int B, size_t* bytes);

/*
 * bsa_backward -- enqueues the gradients of bsa_forward on `stream`.
 *
 * For a loss L with dO = dL/dO, with P the attention weights of the forward
 * (P = exp(scale q_t . k_p - lse_t) on the attended keys, 0 elsewhere):
 *     D_t  = sum_c dO[t,c] O[t,c]
 *     dS   = P (.) (dO V^T - D)                 (the softmax Jacobian)
 *     dQ   = scale dS K,   dK = scale dS^T Q,   dV = P^T dO
 * This is the derivative of the forward's masked attention ("Adapt or Perish:
 * 新手入门指南 – Adaptive Sparse Transformer 核心原理与实战", sparse-attention
 * formula), the training the pages describe ("BERT 稀疏注意力机制入门指南",
 * 生产环境部署建议; "BigBird 稀疏注意力机制解析", 避坑指南) needing it.
 *   q, k, v   device, bf16, [B, H, L, d] contiguous, 16-byte aligned: the
 *             forward's inputs.
 *   out, lse  device: the forward's O (bf16 [B, H, L, d]) and lse (fp32
 *             [B, H, L]) for the same inputs, layout, key_mask and scale.
 *   dout      device, bf16, [B, H, L, d]: dL/dO.
 *   key_mask  device uint8 [B, L] (1 = keep) or NULL, as in the forward.
 *   scale     as in the forward (<= 0 selects 1/sqrt(d)).
 *   dq, dk, dv device, bf16, [B, H, L, d], written in full (zeros for keys no
 *             query attends and for query rows that attend no key).
 *   workspace device, at least bsa_backward_workspace_bytes(layout, B) bytes,
 *             256-byte aligned; no clearing needed.
 * d must be 64 (else BSA_ERR_UNSUPPORTED).  Enqueues up to seven kernels (key
 * bits, D and lse, dQ, dK/dV, and the sums of split tiles for dQ, dK and dV); no
 * synchronisation, no allocation.  A device-side timeout is reported later by
 * bsa_sync_status.
 */
int bsa_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                 const float* lse, int B, int H, int L, int d, const bsa_layout* layout,
                 const uint8_t* key_mask, float scale, void* dq, void* dk, void* dv, void* workspace,
                 size_t workspace_bytes, void* stream);

/*
 * bsa_qkv_projection -- the layer's QKV projection, written in the attention's
 * head layout ("BigBird 稀疏注意力机制解析", 代码实现: self.qkv =
 * nn.Linear(dim, dim * 3), then split into heads).  With C = 64 H:
 *   x     device, bf16 [B, L, C] row-major;
 *   w     device, bf16 [3 C, C] row-major (a linear layer's [out, in] weight):
 *         rows 0..C-1 make q, C..2C-1 k, 2C..3C-1 v; within each, rows
 *         64 h..64 h+63 are head h's 64 features;
 *   bias  device, bf16 [3 C], or NULL for none;
 *   q, k, v  device, bf16 [B, H, L, 64], written:
 *         q[b, h, l, j] = bf16_rne(sum_c x[b, l, c] w[64 h + j, c] + bias[64 h + j])
 *         (k and v with rows C + 64 h + j and 2 C + 64 h + j), fp32 accumulation.
 * All pointers 16-byte aligned; the caller owns every buffer.  B, L, H >= 1
 * (else BSA_ERR_INVALID_ARG).  Enqueues one kernel on `stream` (tcgen05 GEMM,
 * 128 x 256 tiles, the head split done by its stores); no allocation, no
 * synchronisation; a device-side timeout is reported by bsa_sync_status.
 * BSA_ERR_UNSUPPORTED on a device that is not sm_100.
 */
int bsa_qkv_projection(const void* x, const void* w, const void* bias, int B, int L, int H, void* q,
                       void* k, void* v, void* stream);

/*
 * bsa_out_projection -- the layer's output projection over the merged heads
 * ("BERT 稀疏注意力机制入门指南", PyTorch 实现: self.proj = nn.Linear(dim,
 * dim) after the heads are concatenated):
 *   o     device, bf16 [B, H, L, 64] (the attention output);
 *   w     device, bf16 [N, 64 H] row-major (a linear layer's [out, in] weight);
 *   bias  device, bf16 [N], or NULL;
 *   y     device, bf16 [B, L, N], written:
 *         y[b, l, n] = bf16_rne(sum_{h, j} o[b, h, l, j] w[n, 64 h + j] + bias[n]).
 * N a positive multiple of 64 (else BSA_ERR_INVALID_ARG); pointers 16-byte
 * aligned; B, L, H >= 1.  Enqueues one kernel (the heads are merged by the
 * GEMM's own tile loads); no allocation, no synchronisation.
 */
int bsa_out_projection(const void* o, const void* w, const void* bias, int B, int H, int L, int N, void* y,
                       void* stream);

/*
 * bsa_sync_status -- synchronises `stream`, then returns and clears the
 * device-side status word of the current device: BSA_OK, or
 * BSA_ERR_DEVICE_TIMEOUT if a kernel's bounded wait gave up (its outputs are
 * then undefined).  BSA_ERR_CUDA if the synchronisation itself failed.
 */
int bsa_sync_status(void* stream);

/* bsa_strerror -- static description of a status code. */
const char* bsa_strerror(int status);

/*
 * bsa_debug_wait_timeout -- test hook for the bounded-wait machinery: launches
 * one CTA that waits on a shared-memory barrier nothing ever completes, with a
 * limit of `timeout_ns` nanoseconds (clamped to [1e3, 2e9]).  The kernel gives
 * up, records BSA_ERR_DEVICE_TIMEOUT in the status word and returns; the
 * context stays usable.  Read the result with bsa_sync_status.
 */
int bsa_debug_wait_timeout(uint64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
