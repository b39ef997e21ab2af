/*
 * msa.h — C ABI of the B200 (sm_100a) hot path of Memory Sparse Attention (MSA).
 *
 * MSA routes a query over a memory bank of up to 100M tokens: each memory document is
 * encoded once (document-wise RoPE, chunk-mean pooling of K, V and the router key K^R),
 * the pooled router keys stay in GPU memory, the query's router vectors score every chunk
 * by cosine similarity, the top-k documents are selected, their compressed K/V are fetched
 * from host memory and the query attends over them together with its own local K/V. The
 * Memory Interleave loop repeats route -> attend -> append -> re-route.
 *
 * Sources (web pages about the MSA paper, Chen et al., "MSA: Memory Sparse Attention for
 * Efficient End-to-End Memory Model Scaling to 100M Tokens"), cited by tag:
 *   [P1] Lighthouse AI-research news digest of the paper (2026-03-27)
 *   [P2] hotdry blog "EverMind MSA router sparse attention architecture" (2026-03-24)
 *   [P5] wiselychen blog "MSA: 4B 模型打贏 235B RAG 系統"
 *
 * Conventions
 *   - Every call returns msa_status. On failure msa_last_error() gives a thread-local message.
 *   - Validation happens before anything is enqueued: a call that fails validation launches
 *     nothing and copies nothing.
 *   - The caller owns all memory. Device pointers come from the caller's allocator (PyTorch),
 *     pinned host buffers from cudaHostAlloc (torch pin_memory). The library allocates no
 *     device or host memory; scratch space is a caller workspace whose size the matching
 *     *_workspace_size call returns. Tensor memory (TMEM) is allocated and freed inside kernels.
 *   - All calls are asynchronous on the given stream (a cudaStream_t; NULL = legacy default)
 *     unless stated otherwise; outputs are valid once the stream has reached the call.
 *   - Tensors are contiguous and row-major; the layout of each is given with the call.
 *     Device pointers must be 16-byte aligned.
 *   - Kernels that detect a bad value at run time (a position past the RoPE table, a wait
 *     that ran out of time) skip the offending work and record a code in a device-side error
 *     word, read and cleared by msa_device_status(). No kernel traps.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t msa_status;
enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1, /* null or misaligned pointer, bad size, k > n_docs, dtype mismatch */
    MSA_ERR_UNSUPPORTED = 2, /* a shape the kernels do not handle (e.g. head_dim != 128 in attention) */
    MSA_ERR_CUDA = 3,        /* a CUDA runtime or launch error; message in msa_last_error() */
    MSA_ERR_TIMEOUT = 4,     /* a host-side wait passed its deadline */
    MSA_ERR_WORKSPACE = 5,   /* the workspace is smaller than the *_workspace_size answer */
    MSA_ERR_DEVICE = 6       /* a kernel recorded a run-time error (msa_device_status) */
};

typedef int32_t msa_dtype;
enum { MSA_F32 = 0, MSA_BF16 = 1 };

/* Device-side error codes recorded by kernels (first one wins). */
enum {
    MSA_DEV_OK = 0,
    MSA_DEV_ROPE_POSITION = 1, /* a RoPE position was >= max_pos; that row was not rotated/pooled */
    MSA_DEV_WAIT_TIMEOUT = 2,  /* an mbarrier wait in the tensor-core router ran out of time */
    MSA_DEV_BAD_INDEX = 3      /* a doc index outside [0, n_docs) reached a kernel */
};

/* Thread-local text of the last error on this host thread ("" if none). */
const char* msa_last_error(void);

/* Library version string. */
const char* msa_version(void);

/* Synchronises `stream`, then reads and clears the device-side error word of the current
 * device into *code (MSA_DEV_*). Returns MSA_OK, or MSA_ERR_CUDA if the read failed. */
msa_status msa_device_status(int32_t* code, void* stream);

/* Host-only: fills the RoPE table used by every rotating call.
 * out_host is [max_pos][d/2][2] float (cos, sin) of the angle p * base^(-2i/d), computed in
 * double precision by the C math library and rounded once to float. d must be even.
 * ([P1] §组件 2 Document-wise RoPE; rotate-half pairing i <-> i + d/2 with base 1e6 is the
 * reading taken for the Qwen3-like backbone the pages name.) */
msa_status msa_rope_table(int64_t max_pos, int d, double base, float* out_host);

/* Fills chunk_doc[c] = index of the document that owns chunk c, from the CSR offsets
 * doc_chunk_off[n_docs + 1] (device, int64, non-decreasing, doc_chunk_off[n_docs] == n_chunks).
 * chunk_doc is device int32 [n_chunks]. The map is part of the pooled bank's metadata. */
msa_status msa_chunk_doc_map(const int64_t* doc_chunk_off, int64_t n_docs, int64_t n_chunks, int32_t* chunk_doc,
                             void* stream);

/* Rotary position embedding of x [n_tok][n_heads][head_dim] (dt = MSA_F32 or MSA_BF16) into
 * out (same layout; out may equal x for in-place). Token t of segment s (segments given by the
 * device CSR offsets seg_tok_off[n_seg + 1]) gets position pos_offset + (t - seg_tok_off[s]).
 *   Document-wise RoPE of memory keys: one segment per document, pos_offset = 0 — positions
 *   restart at 0 in every document ([P1] §组件 2; [P2] §工程实现的关键细节).
 *   Global RoPE of the active context: one segment per query, pos_offset = k + first local
 *   index — the active context starts at position k, the top-k count ([P1] §组件 2).
 * cos_sin is the device copy of msa_rope_table(max_pos, head_dim, ...). A position >= max_pos
 * leaves that row unrotated in out and records MSA_DEV_ROPE_POSITION.
 * Requires head_dim even, head_dim/VEC a power of two <= 32 (VEC = 4 for fp32, 8 for bf16). */
msa_status msa_rope_doc(const void* x, void* out, msa_dtype dt, int64_t n_tok, int n_heads, int head_dim,
                        const int64_t* seg_tok_off, int64_t n_seg, int64_t pos_offset, const float* cos_sin,
                        int64_t max_pos, void* stream);

/* Offline memory encoding ([P5] §3 inference stage 1; [P2] §可学习记忆路由层的核心架构):
 * chunk-mean pooling of each document's token-level K, V and router key K^R into K-bar, V-bar
 * and K-bar^R. Chunks have `chunk` tokens and never cross a document; a document's last chunk
 * is the mean of its remaining tokens.
 *   k, v: device [n_tok][hkv][d]; kr: device [n_tok][hr][d]; all of dtype in_dt. Any of
 *     (k and v together) or kr may be NULL to skip that part.
 *   doc_tok_off [n_docs+1], doc_chunk_off [n_docs+1]: device int64 CSR offsets (tokens, chunks).
 *   chunk_doc [n_chunks]: device int32 (msa_chunk_doc_map).
 *   fuse_doc_rope: rotate K with document-wise positions (p = token - doc start) before the
 *     mean, using cos_sin [max_pos][d/2][2] (device); K-bar is then the mean of rotated keys.
 *   kvbar: device [n_chunks][2][hkv][d] of out_dt — K-bar at [c][0], V-bar at [c][1] (the
 *     layout of the host content bank, so one document is one contiguous byte run).
 *   kr_index: device [n_chunks][hr][d] of out_dt — K-bar^R; when normalize_router != 0 each
 *     head vector is divided by its L2 norm (a zero vector stays zero): the "index form" that
 *     msa_route_scores reads. Pre-pooled router keys are put into index form by calling this
 *     with chunk = 1, one document per chunk run, k = v = NULL.
 * Arithmetic is fp32 (each element summed in token order); outputs are rounded once to out_dt.
 * Two kernels give the same bits: register streaming (one block per chunk and tensor part) and
 * bulk copy (token rows, and for rotated keys their RoPE table rows, staged in shared memory by
 * cp.async.bulk into a ring of pipeline stages fed by one producer lane; every wait bounded,
 * MSA_DEV_WAIT_TIMEOUT on expiry). By default the bulk-copy kernel runs when chunks x parts is at
 * most two waves of the register kernel's resident blocks, the register kernel otherwise; layouts
 * whose token row exceeds a stage always use the register kernel. */
msa_status msa_pool_chunks(const void* k, const void* v, const void* kr, msa_dtype in_dt, int64_t n_tok, int hkv,
                           int hr, int d, const int64_t* doc_tok_off, const int64_t* doc_chunk_off,
                           const int32_t* chunk_doc, int64_t n_docs, int64_t n_chunks, int chunk, int fuse_doc_rope,
                           const float* cos_sin, int64_t max_pos, void* kvbar, void* kr_index, msa_dtype out_dt,
                           int normalize_router, void* stream);

/* Selects the pooling kernel: 0 = by size (default), 1 = register streaming, 2 = bulk copy where
 * the layout allows. Process-wide. */
msa_status msa_pool_set_impl(int impl);

/* Tuning knob of the bulk-copy pooling kernel: n_stages pipeline stages (2..16) of stage_bytes
 * bytes (a multiple of 1024 in [2048, 65536]), each filled by bulk copies of copy_bytes (a multiple
 * of 16, rounded down to whole token rows, at least one row); 0 keeps the default (3 stages of
 * 32 KiB, one copy per stage). The ring (n_stages * stage_bytes) must stay within 200 KiB.
 * Process-wide. */
msa_status msa_pool_set_pipeline(int n_stages, int stage_bytes, int copy_bytes);

/* Token-level memory bank for the fine stage (coarse-to-fine reading of [P5] 四個核心機制 §1:
 * after routing on the compressed chunks, attention may read the selected documents' own tokens;
 * [P1] §组件 2: memory keys carry document-wise positions). For every token row r of document i
 * (doc_tok_off[i] <= r < doc_tok_off[i+1]):
 *   bank[r][0] = k[r] rotated to position r - doc_tok_off[i];  bank[r][1] = v[r].
 *   k, v: device [n_tok][hkv][d] of dt; doc_tok_off: device int64 [n_docs+1] (doc_tok_off[0] = 0,
 *   doc_tok_off[n_docs] = n_tok); cos_sin: device [max_pos][d/2][2] (msa_rope_table);
 *   bank: device [n_tok][2][hkv][d] of dt — the layout msa_gather_kv and msa_gather_kv_device
 *   read when given doc_tok_off in place of doc_chunk_off, so a document is one contiguous run.
 * A position >= max_pos leaves that key unrotated and records MSA_DEV_ROPE_POSITION.
 * Same head_dim rules as msa_rope_doc. */
msa_status msa_pack_tokens(const void* k, const void* v, msa_dtype dt, int64_t n_tok, int hkv, int d,
                           const int64_t* doc_tok_off, int64_t n_docs, const float* cos_sin, int64_t max_pos,
                           void* bank, void* stream);

/* Router scoring ([P1] §组件 1 key formula; [P2] §可学习记忆路由层的核心架构):
 *   S_{q,c} = max over tokens t of mean over heads h of cos(Q^R_{q,t,h}, K-bar^R_{c,h})
 *   doc_scores[q][i] = max over the chunks c of document i of S_{q,c}
 * (the document score as the max over its chunks is this library's stated reading.)
 *   kr_index: device [n_chunks][H*d] in index form (per-head unit vectors), dtype dt.
 *   qr: device [n_q][T][H][d] raw router queries, dtype dt.
 *   chunk_doc: device int32 [n_chunks]; doc_scores: device float [n_q][n_docs] (output, every
 *   entry written; a document without chunks gets -inf); chunk_scores: device float
 *   [n_q][n_chunks] or NULL.
 * The mean of the per-head cosines is computed as one dot product: each query head vector is
 * divided by its norm and by H, the heads are concatenated, and the dot product with the
 * concatenated unit-vector index row is the mean of the cosines. bf16 runs on the tcgen05
 * tensor cores (fp32 accumulation in TMEM) when H*d % 64 == 0; fp32 runs on CUDA cores in
 * fp32. ws: device workspace of msa_route_workspace_size bytes (256-byte aligned). */
msa_status msa_route_scores(const void* kr_index, msa_dtype dt, int64_t n_chunks, const int32_t* chunk_doc,
                            int64_t n_docs, const void* qr, int n_q, int T, int H, int d, float* doc_scores,
                            float* chunk_scores, void* ws, size_t ws_bytes, void* stream);
msa_status msa_route_workspace_size(int n_q, int T, int H, int d, msa_dtype dt, size_t* bytes);

/* Selects the router kernel for testing: 0 = automatic, 1 = CUDA-core kernel, 2 = tensor-core
 * kernel (bf16 only; the normalised queries stream from L2 with every index tile), 3 = tensor-core
 * kernel with the normalised queries held in shared memory when they fit. Process-wide. */
msa_status msa_route_set_impl(int impl);

/* Tuning knob of the tensor-core router: at most n pipeline stages of index tiles (1 <= n <= 12;
 * 0 = default, as many as fit in a shared-memory budget that leaves each SM room for one
 * attention block and one top-k block running concurrently). Process-wide. */
msa_status msa_route_set_max_stages(int n);

/* Failure-detection test hook of the tensor-core router: while on, each launch's producer
 * publishes no tile and issues no copy, so the other warps' bounded waits expire (about 2 s); the
 * kernel then records MSA_DEV_WAIT_TIMEOUT, frees its tensor memory and returns, leaving the
 * context usable. Scores written by such launches are meaningless. Process-wide. */
msa_status msa_route_inject_stall(int on);

/* Top-k document selection ([P1] §组件 1; [P2] Top-k 选择机制): for every query the k documents
 * with the largest doc_scores, in descending score order, ties broken by the lower document
 * index. doc_scores: device float [n_q][n_docs]; idx: device int32 [n_q][k]; score: device
 * float [n_q][k] (may be NULL). 1 <= k <= min(64, n_docs). ws: msa_topk_workspace_size bytes. */
msa_status msa_topk_docs(const float* doc_scores, int n_q, int64_t n_docs, int k, int32_t* idx, float* score,
                         void* ws, size_t ws_bytes, void* stream);
msa_status msa_topk_workspace_size(int n_q, int64_t n_docs, int k, size_t* bytes);

/* Allocation-free variant of msa_topk_docs. The pages have no counterpart: this is a library
 * addition for callers that cannot allocate device memory when they select documents — a host
 * application that loads this library as a plugin and hands it only its own input and output
 * buffers, a serving loop whose device memory is reserved up front by its own pool, or a
 * latency-bound loop that cannot take cudaMalloc's implicit device synchronisation.
 * Same arguments and results as msa_topk_docs without the workspace: the scratch (partial lists
 * and ticket counters) is a fixed array of msa_topk_noalloc_max_scratch() bytes (1 MiB) in the
 * library's device memory, held by every GPU that loads the library until the process exits.
 * A size whose scratch (msa_topk_workspace_size) exceeds it fails with MSA_ERR_INVALID_ARG and
 * launches nothing. The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream capture. Every call
 * shares the array: calls whose work overlaps on the GPU (other streams, other host threads on
 * the same device) race and corrupt each other's results, so order them on one stream. Calls no
 * cudaMalloc, cudaFree or allocating library routine. */
msa_status msa_topk_docs_noalloc(const float* doc_scores, int n_q, int64_t n_docs, int k, int32_t* idx, float* score,
                                 void* stream);
size_t msa_topk_noalloc_max_scratch(void);

/* Memory Parallel merge ([P2] §工程实现的关键细节: the router keys are sharded over several GPUs,
 * each scores its own keys and keeps its local best, and the local results are combined into the
 * global top-k; [P3] §四大技术突破 3). Shard g holds the documents
 * shard_doc_off[g] .. shard_doc_off[g+1]-1 and supplies its local top-k_cand list.
 *   cand_score, cand_idx: device float / int32 lists [n_q][k_cand] of every shard, shard g's lists
 *     starting shard_stride * g elements after cand_score / cand_idx (n_q * k_cand for two plain
 *     [n_shards][n_q][k_cand] arrays; 2 * n_q * k_cand when every rank packed [scores ; indices]
 *     into one buffer and an all_gather concatenated them). Indices are local to their shard, -1
 *     for an empty slot;
 *   shard_doc_off: HOST int64 [n_shards+1], non-decreasing;
 *   idx: device int32 [n_q][k]: the k best candidates as GLOBAL document indices, by descending
 *     score, equal scores to the lower global index (-0 equals +0, a NaN score ranks below -inf);
 *     score: device float [n_q][k] (may be NULL). Slots past the number of candidates hold -1 and
 *     -inf. With disjoint shards whose lists are their exact local top-k (k_cand >= k) the result is
 *     exactly msa_topk_docs over all documents.
 * Requires 1 <= n_shards <= 64, n_shards * k_cand <= 4096, 1 <= k <= 64, global indices < 2^31.
 * A local index outside its shard (other than -1) records MSA_DEV_BAD_INDEX and counts as empty.
 * Duplicate candidates are not removed. One block per query. */
msa_status msa_topk_merge(const float* cand_score, const int32_t* cand_idx, int64_t shard_stride, int n_shards,
                          int n_q, int k_cand, const int64_t* shard_doc_off, int k, int32_t* idx, float* score,
                          void* stream);

/* Fetch of the selected documents' compressed K-bar/V-bar from host memory
 * ([P2] §工程实现的关键细节: K-bar^R stays in GPU memory, K-bar/V-bar live in host DRAM and are
 * loaded asynchronously once routing has chosen the documents; [P5] §3 async prefetch).
 *   host_bank: pinned host [n_chunks][2][hkv][d] of dt (the kvbar layout of msa_pool_chunks).
 *   doc_chunk_off_host: host int64 [n_docs+1]; idx_host: host int32 [n_q][k] (msa_topk_docs
 *   output copied to the host).
 *   dev_mem_kv: device [n_q][max_mem][2][hkv][d]: query q's selected documents' chunk rows,
 *   concatenated in rank order from row 0; mem_len_host[q] (host int32, written before the
 *   call returns) is the number of rows filled.
 * One cudaMemcpyAsync per selected document on copy_stream (the copy engines over the host
 * link); the call returns once they are enqueued. The fine stage passes the token bank of
 * msa_pack_tokens with doc_tok_off in place of doc_chunk_off (rows are then tokens). Fails with MSA_ERR_INVALID_ARG, copying
 * nothing, if an index is out of range or a query's rows exceed max_mem. */
msa_status msa_gather_kv(const void* host_bank, msa_dtype dt, int64_t n_chunks, const int64_t* doc_chunk_off_host,
                         int64_t n_docs, const int32_t* idx_host, int n_q, int k, int hkv, int d, int max_mem,
                         void* dev_mem_kv, int32_t* mem_len_host, void* copy_stream);

/* Device-side variant of msa_gather_kv: a kernel on `stream` reads the selected documents' rows
 * straight from the pinned host bank (mapped into the device address space; the pointer must come
 * from cudaHostAlloc / torch pin_memory) with device-resident indices, so no host round trip sits
 * between selection and fetch. Same layout and rank order as msa_gather_kv. A bank in the current
 * device's own memory (a training context) is accepted too and read directly.
 *   doc_chunk_off: device int64 [n_docs+1]; idx: device int32 [n_q][k]; mem_len: device int32 [n_q].
 * Indices out of range or more rows than max_mem record MSA_DEV_BAD_INDEX and skip that query's
 * copy (no out-of-range access). Long documents (token rows of the fine stage) are split over
 * several blocks, chosen from max_mem / k. Returns MSA_ERR_INVALID_ARG if host_bank is neither device memory nor pinned, mapped
 * host memory. */
msa_status msa_gather_kv_device(const void* host_bank, msa_dtype dt, int64_t n_chunks, const int64_t* doc_chunk_off,
                                int64_t n_docs, const int32_t* idx, int n_q, int k, int hkv, int d, int max_mem,
                                void* dev_mem_kv, int32_t* mem_len, void* stream);

/* Sparse attention ([P1] §组件 1 稀疏注意力机制; [P2] concatenation of the selected compressed
 * K/V with the query's local K/V): for query q, token t, head h (kv head g = h / (hq/hkv)):
 *   out = softmax(scale * q . [mem K-bar ; local K_j, j <= q_start + t, j < L]) [mem V-bar ; local V]
 *   q: device [n_q][T][hq][d], already rotated (global positions);
 *   mem_kv: device [n_q][max_mem][2][hkv][d] (msa_gather_kv), mem_len: device int32 [n_q];
 *   local_k, local_v: device [n_q][L_max][hkv][d], rotated keys of the active context;
 *   out: device [n_q][T][hq][d]. All of dtype dt; arithmetic and softmax in fp32.
 * Memory rows are all visible; local keys are causal. A row with no visible key is 0.
 * bf16 runs on tensor cores (mma.sync, fp32 accumulation), fp32 on CUDA cores.
 * Requires d == 128 and hq/hkv in {1, 2, 4, 8}. */
msa_status msa_sparse_attn(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem,
                           const void* local_k, const void* local_v, int L_max, int L, int q_start, int n_q, int T,
                           int hq, int hkv, int d, float scale, void* out, msa_dtype dt, void* stream);

/* Selects the bf16 attention kernels for testing: 0 = default (msa_sparse_attn_split on tcgen05
 * tensor cores with TMEM accumulators, msa_sparse_attn on mma.sync m16n8k16 so that it can run
 * beside the router's blocks), 1 = CUDA cores for msa_sparse_attn, 2 = mma.sync for both,
 * 3 = as 0, and the attention backward's dK / dV on tcgen05 as well (by default they run on
 * mma.sync, dQ on tcgen05). impl 3 has not yet been validated on a GPU: opt-in only.
 * fp32 always runs on CUDA cores. Process-wide. */
msa_status msa_attn_set_impl(int impl);

/* Sparse attention over long memories (the token-level fine stage, thousands of memory rows per
 * query): the same arguments, layout and result as msa_sparse_attn, computed with the keys of
 * every row block (of kv head g and query q) split into n_split contiguous ranges of 64-key tiles
 * that run as separate blocks. Default (msa_attn_set_impl(0)): tcgen05 tensor cores, one CTA of
 * 192 threads per 128 (token, head) rows and key range, S and O accumulated in TMEM, K/V tiles of
 * memory rows and of local keys loaded by TMA; n_split sized for one wave of one CTA per SM (148
 * SMs). impl 2: mma.sync, 64-row blocks, one wave of three blocks per SM. Ranges hold at least
 * four tiles. Each range writes its unnormalised output and (running max, sum) in fp32 to the
 * workspace; a second kernel merges the ranges' softmax statistics and writes out.
 * bf16 only (tensor cores); fp32 returns MSA_ERR_UNSUPPORTED.
 * lse: optional device float [n_q][T][hq]: ln sum_j exp(scale * q . k_j) over the row's visible
 * keys (-inf for a row without one), what msa_sparse_attn_backward needs from the forward pass.
 * ws: device, msa_sparse_attn_split_workspace_size bytes, 16-byte aligned. */
msa_status msa_sparse_attn_split(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem,
                                 const void* local_k, const void* local_v, int L_max, int L, int q_start, int n_q,
                                 int T, int hq, int hkv, int d, float scale, void* out, float* lse, msa_dtype dt,
                                 void* ws, size_t ws_bytes, void* stream);
msa_status msa_sparse_attn_split_workspace_size(int n_q, int T, int hq, int hkv, int max_mem, int L, size_t* bytes);

/* The launch plan msa_sparse_attn_split would use on the current device for these sizes (a query:
 * enqueues nothing). *row_blocks: 128-row blocks per tensor-core CTA (1 or 2; 0 on the mma.sync
 * path); *key_ranges: key ranges per (row blocks, kv head, query); *cluster: when >= 1, the ranges
 * form a thread-block cluster of that many CTAs and are merged in distributed shared memory (no
 * combine pass), 0 when partial results are combined through the workspace. */
msa_status msa_sparse_attn_split_plan(int n_q, int T, int hq, int hkv, int max_mem, int L, int* row_blocks,
                                      int* key_ranges, int* cluster);

/* ---------------------------------------------------------------------------------------------
 * Backward pass (end-to-end training: [P1] 核心创新 端到端可训练性 — routing, compression and
 * attention are optimised in one gradient flow; [P1] §训练策略 and [P2] §训练层面 — a weighted
 * auxiliary loss supervises every layer's router). The top-k selection carries no gradient. All
 * gradients are fp32; device pointers; calls are asynchronous on `stream`.
 * --------------------------------------------------------------------------------------------- */

/* Gradients of msa_sparse_attn / msa_sparse_attn_split with respect to q, the fetched memory and
 * the local K/V, given dout = dL/dout. Same layouts and sizes as the forward; out (bf16) and
 * lse (msa_sparse_attn_split's log-sum-exp) come from the forward pass.
 *   dq: [n_q][T][hq][d]; dmem_kv: [n_q][max_mem][2][hkv][d] (rows < mem_len[q] written);
 *   dlocal_k, dlocal_v: [n_q][L_max][hkv][d] (rows < L written). All overwritten, not added to.
 * For each row, with P the softmax of the forward: dV = P^T dO, dS = P * (dO V^T - rowsum(dO*O)),
 * dq = scale dS K, dK = scale dS^T q, summed over the query heads that share a kv head. Tensor
 * cores (mma.sync, bf16 operands: P and dS are rounded to bf16, fp32 accumulation); each key's
 * gradient is accumulated over contiguous ranges of rows by as many blocks as fill about one wave,
 * the ranges' partial sums then added in a fixed order (deterministic, no atomics). bf16 only,
 * d == 128, hq/hkv in {1, 2, 4, 8}. ws: msa_sparse_attn_backward_workspace_size bytes. */
msa_status msa_sparse_attn_backward(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem,
                                    const void* local_k, const void* local_v, int L_max, int L, int q_start, int n_q,
                                    int T, int hq, int hkv, int d, float scale, const void* out, const void* dout,
                                    const float* lse, msa_dtype dt, float* dq, float* dmem_kv, float* dlocal_k,
                                    float* dlocal_v, void* ws, size_t ws_bytes, void* stream);
msa_status msa_sparse_attn_backward_workspace_size(int n_q, int T, int hq, int hkv, int max_mem, int L,
                                                   size_t* bytes);

/* Adjoint of the fetch (msa_gather_kv_device): query q's memory-row gradients dmem_kv
 * [n_q][max_mem][2][hkv][d] (fp32) are added to the chunk rows of dkvbar [n_chunks][2][hkv][d]
 * (fp32) they were copied from, following idx [n_q][k] and doc_chunk_off (device) in rank order;
 * a document selected by several queries receives the sum (fp32 atomic adds, so the summation
 * order varies). With accumulate == 0 dkvbar is zeroed first (on the stream), else added to.
 * Bad indices record MSA_DEV_BAD_INDEX and are skipped. */
msa_status msa_gather_kv_backward(const float* dmem_kv, int64_t n_chunks, const int64_t* doc_chunk_off,
                                  int64_t n_docs, const int32_t* idx, int n_q, int k, int hkv, int d, int max_mem,
                                  float* dkvbar, int accumulate, void* stream);

/* Adjoint of msa_pool_chunks: token gradients from chunk gradients.
 *   dkvbar: fp32 [n_chunks][2][hkv][d] (dK-bar, dV-bar) or NULL; then dk, dv: fp32 [n_tok][hkv][d]
 *     with dk[t] = R(-p_t) dK-bar[c] / n_c (p_t the token's position in its document; without
 *     fuse_doc_rope no rotation) and dv[t] = dV-bar[c] / n_c for every token t of chunk c (n_c tokens).
 *   dkr_index: fp32 [n_chunks][hr][d] or NULL, the gradient with respect to the stored router index;
 *     then dkr: fp32 [n_tok][hr][d]. With normalize_router the index was unit(K-bar^R) per head and
 *     the gradient passes through the normalisation, (g - k_hat (k_hat . g)) / |K-bar^R|, the raw
 *     chunk mean K-bar^R being recomputed from kr (token K^R [n_tok][hr][d] of kr_dt); without it
 *     kr may be NULL. Needs hr * d <= 1024 and (normalised) d a multiple of 32 up to 256.
 * Offsets, table and chunking as for msa_pool_chunks. */
msa_status msa_pool_chunks_backward(const float* dkvbar, const float* dkr_index, const void* kr, msa_dtype kr_dt,
                                    int64_t n_tok, int hkv, int hr, int d, const int64_t* doc_tok_off,
                                    const int64_t* doc_chunk_off, const int32_t* chunk_doc, int64_t n_docs,
                                    int64_t n_chunks, int chunk, int fuse_doc_rope, const float* cos_sin,
                                    int64_t max_pos, int normalize_router, float* dk, float* dv, float* dkr,
                                    void* stream);

/* Auxiliary router loss and its gradient (reading of [P1] §训练策略 辅助损失, which states the
 * supervision but no formula): for query q with evidence documents E_q (evidence [n_q][n_ev] int32,
 * -1 = padding), s = doc_scores[q] / tau,
 *   loss[q] = -(1/|E_q|) sum_{e in E_q} (s_e - log sum_i exp s_i)      (loss may be NULL)
 *   d_doc_scores[q][i] = (softmax(s)_i - [i in E_q] / |E_q|) / tau / n_q
 * i.e. the gradient of the mean of loss[] over the queries. One block per query. */
msa_status msa_router_aux_loss(const float* doc_scores, int n_q, int64_t n_docs, const int32_t* evidence, int n_ev,
                               float tau, float* loss, float* d_doc_scores, void* stream);

/* Gradients of msa_route_scores' document scores given d_doc_scores [n_q][n_docs] (fp32):
 * each document's score is attained at one (chunk, query token) pair — the first chunk, then the
 * first token, on exact ties — and only that pair receives its gradient:
 *   dqr [n_q][T][H][d] (fp32): with respect to the raw router queries, through their per-head
 *     normalisation;
 *   dkhat [n_chunks][H][d] (fp32, overwritten): with respect to the stored index vectors as used
 *     in the dot product (msa_pool_chunks_backward carries it through the index normalisation).
 * Scores are recomputed to find the attaining pairs (a training-context bank, not the 100M
 * inference index): for a bf16 index with H * d a multiple of 64, on the tcgen05 tensor cores with
 * the fp32 normalised queries split exactly into three bf16 terms (fp32 accumulation in TMEM;
 * msa_route_set_impl(1) selects the CUDA-core search instead); otherwise in fp32 on CUDA cores.
 * kr_index and qr of dtype dt; H * d <= 1024.
 * ws: msa_route_backward_workspace_size bytes (device, 256-byte aligned). */
msa_status msa_route_backward(const void* kr_index, msa_dtype dt, int64_t n_chunks, const int64_t* doc_chunk_off,
                              int64_t n_docs, const void* qr, int n_q, int T, int H, int d, const float* d_doc_scores,
                              float* dqr, float* dkhat, void* ws, size_t ws_bytes, void* stream);
msa_status msa_route_backward_workspace_size(int64_t n_chunks, int n_q, int T, int H, int d, size_t* bytes);

/* One routed layer of one Memory Interleave round (see msa_interleave_step). */
typedef struct msa_layer_args {
    const void* kr_index;       /* device [n_chunks][H*d], index form */
    const void* host_bank;      /* pinned host [n_chunks][2][hkv][d] */
    const void* qr;             /* device [n_q][T_act][H][d]: router queries of every active token */
    const void* q_new;          /* device: raw queries of the tokens appended this round,
                                   element (q, t, h, i) at ((q * new_q_stride + t) * hq + h) * d + i */
    const void* k_new;          /* device: raw keys of the appended tokens, same indexing with hkv */
    const void* v_new;          /* device: values of the appended tokens, same indexing with hkv */
    void* local_k;              /* device [n_q][L_max][hkv][d]: rotated local keys (appended here) */
    void* local_v;              /* device [n_q][L_max][hkv][d] */
    void* out;                  /* device [n_q][T_new][hq][d]: attention output of the appended tokens */
    int32_t* topk_idx_host;     /* pinned host [n_q][k]: documents selected for this layer (output) */
} msa_layer_args;

typedef struct msa_interleave_args {
    int n_layers;
    const msa_layer_args* layers;   /* host array [n_layers] */
    msa_dtype dt;                   /* MSA_BF16 or MSA_F32, for every tensor */
    int64_t n_chunks, n_docs;
    const int64_t* doc_chunk_off;   /* device int64 [n_docs+1] */
    const int64_t* doc_chunk_off_host; /* host int64 [n_docs+1] */
    const int32_t* chunk_doc;       /* device int32 [n_chunks] */
    int n_q, H, d, hq, hkv, k;
    int L_prev;                     /* tokens each query held before this round */
    int T_new;                      /* tokens appended this round (T_act = L_prev + T_new) */
    int new_q_stride;               /* tokens per query in the q_new/k_new/v_new buffers */
    int L_max;                      /* capacity of local_k/local_v per query */
    int max_mem;                    /* capacity of the gathered memory per query (rows) */
    const float* rope_cos_sin;      /* device table of msa_rope_table(rope_max_pos, d, base) */
    int64_t rope_max_pos;
    float scale;                    /* attention scale, normally 1/sqrt(d) */
    int reserved_sms;               /* SMs the router kernels leave free for the overlapped selection
                                       and attention of earlier layers (0 = routers use every SM) */
    void* const* route_events;      /* optional (NULL = none): 2 * n_layers cudaEvent_t created by the
                                       caller; [2l] and [2l+1] are recorded on `compute` just before and
                                       after layer l's router kernel, to time it inside the round */
    int fetch_mode;                 /* 0: the host waits for each layer's selection and issues one
                                       cudaMemcpyAsync per document on `copy` (msa_gather_kv);
                                       1: a device kernel fetches from the mapped pinned bank right
                                       after selection (msa_gather_kv_device), no host waits */
    void* ws;                       /* device workspace of msa_interleave_workspace_size bytes */
    size_t ws_bytes;
} msa_interleave_args;

/* One Memory Interleave round over every routed layer ([P1] §组件 3 Memory Interleaving;
 * [P2] re-route with the updated context each round; [P5] §4 生成式檢索 -> 上下文擴展 -> 生成 ->
 * 再檢索). Per layer: append the round's T_new tokens to the local cache (keys rotated to
 * global positions k + L_prev + t, values copied), rotate their queries likewise, score the
 * memory with the router queries of all T_act = L_prev + T_new active tokens, select the top-k
 * documents, copy their indices to topk_idx_host, fetch their K-bar/V-bar from the host bank on
 * `copy` and attend. The router kernels run back to back on `compute`; selection and attention
 * run on two library-owned streams (created once per device) that fork from and join back into
 * `compute`, so a layer's selection, fetch and attention overlap the routing of later layers.
 * With fetch_mode 0 the host waits for each layer's selection (polling with a deadline of
 * host_wait_timeout_us, giving MSA_ERR_TIMEOUT) before enqueueing its copies; with fetch_mode 1
 * the fetch is a device kernel and the call never waits. When the call returns, everything is
 * enqueued and `compute` is ordered after all of it. */
msa_status msa_interleave_step(const msa_interleave_args* a, void* compute, void* copy, int64_t host_wait_timeout_us);
msa_status msa_interleave_workspace_size(const msa_interleave_args* a, size_t* bytes);

/* The same round captured once into a CUDA graph and replayed: the launches, copies and stream
 * fork/join of msa_interleave_step with fetch_mode 1 (the only mode without host waits), recorded
 * against the buffers and sizes that `a` names at creation. A replay reads whatever those buffers
 * hold when it runs, so a caller refills the round's inputs (qr, q_new, k_new, v_new) in place
 * between replays; everything else in `a` is fixed for the graph's lifetime. Replaying replaces
 * the round's per-launch host work (argument checks, tensor maps, plans, about 10 launches per
 * layer) with one graph launch, which is what bounds short rounds.
 * create: a->fetch_mode must be 1 and a->route_events NULL (MSA_ERR_INVALID_ARG otherwise);
 * `stream` must be a created stream, not the legacy default stream (MSA_ERR_INVALID_ARG). It runs
 * the round once on `stream` (settling one-time set-up: library streams, events, kernel
 * attributes), waits for it, then captures a second pass without executing it. On failure nothing
 * is returned in *out and the capture is ended. The graph is tied to the device current at
 * creation. launch: enqueues one replay on `stream`; `stream` is ordered after all of it when the
 * call returns. destroy: releases the graph; call it once no replay is pending (NULL is a no-op). */
typedef struct msa_interleave_graph msa_interleave_graph;
msa_status msa_interleave_graph_create(const msa_interleave_args* a, void* stream, msa_interleave_graph** out);
msa_status msa_interleave_graph_launch(msa_interleave_graph* g, void* stream);
msa_status msa_interleave_graph_destroy(msa_interleave_graph* g);

/* ----------------------------------------------------------------------------------------------
 * One workspace query for every call that takes a workspace. op names the call, cfg points to the
 * matching configuration struct below (host memory, read only), *bytes receives the size that
 * call needs (the same answer as its own *_workspace_size function, which stays available).
 * Unknown op, NULL cfg or NULL bytes: MSA_ERR_INVALID_ARG; sizes the call itself would refuse:
 * the same status as its *_workspace_size. Host-only, enqueues nothing. The pages define no
 * interface; the query exists because the caller owns all scratch memory.
 * ---------------------------------------------------------------------------------------------- */
enum {
    MSA_OP_ROUTE = 1,               /* msa_route_scores          cfg: const msa_route_ws_cfg*     */
    MSA_OP_TOPK = 2,                /* msa_topk_docs             cfg: const msa_topk_ws_cfg*      */
    MSA_OP_SPARSE_ATTN_SPLIT = 3,   /* msa_sparse_attn_split     cfg: const msa_attn_ws_cfg*      */
    MSA_OP_SPARSE_ATTN_BACKWARD = 4,/* msa_sparse_attn_backward  cfg: const msa_attn_ws_cfg*      */
    MSA_OP_ROUTE_BACKWARD = 5,      /* msa_route_backward        cfg: const msa_route_bwd_ws_cfg* */
    MSA_OP_INTERLEAVE = 6           /* msa_interleave_step       cfg: const msa_interleave_args*  */
};
typedef struct { int n_q, T, H, d; msa_dtype dt; } msa_route_ws_cfg;
typedef struct { int n_q; int64_t n_docs; int k; } msa_topk_ws_cfg;
typedef struct { int n_q, T, hq, hkv, max_mem, L; } msa_attn_ws_cfg;
typedef struct { int64_t n_chunks; int n_q, T, H, d; } msa_route_bwd_ws_cfg;
msa_status msa_workspace_size(int op, const void* cfg, size_t* bytes);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
