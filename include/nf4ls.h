/*
 * nf4ls.h -- C ABI of the layer-streamed NF4 QLoRA training library (libnf4ls.so).
 *
 * What the library computes comes from the pages on layer-streamed NF4 QLoRA
 * training of the "Soup" project, cited here by page title and section:
 *
 *   [gate]   "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
 *            (m.mzlw.cn): §1.3 resident-NF4 reference, §2.1 offline shards and per-call views, §2.2 the six
 *            correctness checks, §2.4 bytes per weight and constant code tables,
 *            §4.3 resident embedding / lm_head, §4.4 the C=6 / C=4 FLOP convention.
 *   [review] "4GB 显存微调 8B 模型是真的：拆解 Soup 的 layer streaming" and its English
 *            version "Fine-Tune 8B Models on 4GB VRAM: Soup's Layer Streaming"
 *            (tools.cooconsbit.com): mechanism section (pinned host store, 2-8 HBM
 *            buffers, side-stream prefetch of layer i+1 forward / i-1 backward,
 *            forced checkpointing, dL/dx = W^T dL/dy), bug history (Issue #331,
 *            pooled-buffer aliasing above ~165 MiB layers).
 *
 * Conventions for every call:
 *   - Return value: NF4LS_OK (0) or a negative status below.  nf4ls_last_error()
 *     returns a thread-local message for the last failure.  No C++ exception
 *     crosses this boundary.
 *   - Pointers named *_dev are device (HBM) pointers; *_host are host pointers.
 *     The caller owns all device and pinned memory and all streams.  The library
 *     never allocates device memory; it owns only CUDA events, the pool's copy
 *     stream and host bookkeeping.  Scratch is passed in as a workspace whose size
 *     a *_bytes() query returns.
 *   - Work is enqueued on the given stream (nf4ls_stream = cudaStream_t) and the
 *     calls return without synchronising.  An asynchronous kernel fault surfaces at
 *     the caller's next synchronisation; a kernel whose bounded wait expired
 *     records it in a device flag that nf4ls_device_error() reads.
 *   - bf16 tensors are row-major with the last dimension contiguous.  Token-major
 *     activations are [M, features] with M = batch * seq, sequences contiguous.
 *   - Device pointers must be 16-byte aligned (NF4LS_ALIGN otherwise); shards and
 *     workspaces 256-byte aligned.
 */
#ifndef NF4LS_H
#define NF4LS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */
#define NF4LS_OK                    0
#define NF4LS_INVALID_ARG          -1  /* null pointer, bad enum, size out of range   */
#define NF4LS_SHAPE                -2  /* dimensions the kernels do not support       */
#define NF4LS_ALIGN                -3  /* pointer or size misaligned                  */
#define NF4LS_CODEBOOK_MISMATCH    -4  /* shard built with other code tables ([gate] §2.4) */
#define NF4LS_FINGERPRINT_MISMATCH -5  /* shard of another checkpoint ([review] cache key)  */
#define NF4LS_BUFFER_BUSY          -6  /* every pool slot is acquired                 */
#define NF4LS_TIMEOUT              -7  /* a bounded host wait expired                 */
#define NF4LS_CUDA                 -8  /* a CUDA runtime call failed                  */
#define NF4LS_DEVICE_FAULT         -9  /* a kernel's bounded wait expired             */
#define NF4LS_SOURCE_REFUSED      -10  /* a stream source too slow, or a SATA / spinning
                                          disk ([review] mechanism: refused outright)   */
#define NF4LS_IO                  -11  /* a file read failed                          */

typedef void* nf4ls_stream; /* cudaStream_t */

const char* nf4ls_last_error(void);
int nf4ls_version(void);

/* Number of kernels the library has launched in this process (all devices). */
uint64_t nf4ls_launch_count(void);

/* Per-launch timing with CUDA events recorded on the launching stream (off by
 * default): every GEMM launch and the phases of the model step.  nf4ls_profile_read
 * waits for the matching records and returns out[0] = count, out[1] = total ms,
 * out[2] = total algorithmic FLOPs (2 M N K per GEMM launch).  sel < 1000 selects a
 * kind (0 dense bf16 GEMM, 1 NF4-decode GEMM, 2 step phase); sel >= 1000 a detail:
 * 1000 + 100 * (NF4 decode) + 10 * (dL/dx product) + epilogue (0 store, 1 residual,
 * 2 RoPE, 3 SwiGLU, 4 SwiGLU backward) for GEMMs, and 2000 layer forwards, 2001
 * final norm + lm_head + loss, 2002 lm_head dL/dx + final-norm backward, 2003 layer
 * backwards for phases.  nf4ls_profile_reset forgets every record. */
int nf4ls_profile(int on);
int nf4ls_profile_read(int sel, double out[3]);
int nf4ls_profile_reset(void);

/* Reads and clears the device error flag of the current device: out[0] = code
 * (0 none, 1 barrier timeout), out[1] = kernel id, out[2] = block, out[3] = site.
 * Synchronises the device. */
int nf4ls_device_error(int32_t out[4]);

/* Exercises the expiry of a bounded wait, the path a kernel takes instead of
 * hanging when an arrival it waits for never comes.  Launches one block of two warps
 * on `stream` that wait on an mbarrier nothing arrives on: warp 0 gives up after
 * limit_us microseconds and records code 1, kernel id 3, block 0, site 1 in the
 * device error record; warp 1 (limit 1000x longer) leaves through the abort flag
 * that warp 0 raised.  result_dev: 2 int32 (device), set to 0 for each warp whose
 * wait did not complete.  The kernel ends by itself; the context stays usable.
 * NF4LS_INVALID_ARG for limit_us outside [1, 1e6] or a NULL result.  No passage of
 * the pages defines this: it is the library's own failure detection. */
int nf4ls_wait_probe(int32_t limit_us, int32_t* result_dev, nf4ls_stream stream);

/* ------------------------------------------------------------------ code tables
 * [gate] §2.4: the NF4 code table (16 fp32) and the nested absmax table (256 fp32)
 * are constant for every weight, so one resident copy is shared; the shard records
 * their hash and the library refuses a shard built with other tables.
 * The library builds both from the published constructions (QLoRA NormalFloat,
 * Dettmers 2023; signed dynamic tree quantisation, Dettmers 2016) in float64,
 * rounded once to fp32, and returns them with their FNV-1a 64-bit hash (over the
 * little-endian fp32 bytes of nf4 then code8).  Any output pointer may be NULL. */
int nf4ls_codebooks(float nf4_host[16], float code8_host[256], uint64_t* hash);

/* ------------------------------------------------------------------ layer config */
typedef struct {
    int32_t hidden;      /* H                                   */
    int32_t inter;       /* I (SiLU-gated MLP width)            */
    int32_t n_q;         /* query heads                         */
    int32_t n_kv;        /* key/value heads (GQA)               */
    int32_t head_dim;    /* d: 64 or 128                        */
    int32_t batch;       /* sequences per step                  */
    int32_t seq;         /* tokens per sequence; M = batch*seq  */
    float rope_theta;    /* RoPE base                           */
    float rms_eps;       /* RMSNorm epsilon                     */
    int32_t lora_r;      /* LoRA rank (16)                      */
    float lora_alpha;    /* LoRA alpha (32); scale = alpha / r  */
} nf4ls_layer_cfg;

/* Tensor kinds of a layer shard, in shard order. */
#define NF4LS_T_Q         0
#define NF4LS_T_K         1
#define NF4LS_T_V         2
#define NF4LS_T_O         3
#define NF4LS_T_GATE      4
#define NF4LS_T_UP        5
#define NF4LS_T_DOWN      6
#define NF4LS_T_NORM_IN   7
#define NF4LS_T_NORM_POST 8
#define NF4LS_N_TENSORS   9

/* ------------------------------------------------------------------ NF4 tensors
 * One frozen linear W [rows, cols] (row-major bf16, rows = out features) in the
 * double-quantised NF4 format of [gate] §2.1/§2.4, n = rows*cols, n % 64 == 0:
 *   packed  u8  [n/2]              code of element 2j in the high nibble of byte j,
 *                                  element 2j+1 in the low nibble
 *   q8      u8  [n/64]             8-bit code of (absmax_b - offset) / nested_g
 *   nested  f32 [ceil(n/16384)]    max |absmax_b - offset| over 256 blocks
 *   offset  f32 [1]                mean of the fp32 absmax values
 * i.e. n/2 + n/64 + 4*ceil(n/16384) + 4 bytes, about 0.516 B/param.
 * Quantisation: absmax_b = max |w| over block b of 64; code = nearest NF4 entry to
 * fp32(w / absmax_b) (midpoint rule, ties to the lower index; absmax 0 -> the
 * exact-zero code); offset = fp32(sequential float64 sum of absmax / count);
 * q8 = nearest code8 entry to fp32((absmax_b - offset) / nested_g).
 * Dequantisation: s_b = fp32(fp32(code8[q8_b] * nested_g) + offset);
 * w^ = bf16_rne(fp32(nf4[code] * s_b)); no fused multiply-add.
 *
 * nf4_quantize_tensor: w_dev bf16 [n] -> packed/q8/nested/offset (device).  Needs
 * scratch_dev of nf4ls_quantize_scratch_bytes(n) bytes.  Deterministic: the same
 * input gives the same bytes on every call.
 * nf4_dequantize_tensor: the inverse map to bf16 out_dev [n] (the standalone,
 * HBM-bound dequantiser; the GEMMs decode inside their mainloop instead). */
size_t nf4ls_quantize_scratch_bytes(size_t n);
int nf4_quantize_tensor(const void* w_dev, size_t n, uint8_t* packed_dev, uint8_t* q8_dev,
                        float* nested_dev, float* offset_dev, void* scratch_dev,
                        size_t scratch_bytes, nf4ls_stream stream);
int nf4_dequantize_tensor(const uint8_t* packed_dev, const uint8_t* q8_dev, const float* nested_dev,
                          const float* offset_dev, size_t n, void* out_dev, nf4ls_stream stream);

/* nf4_quantize_tensor without a scratch argument, for callers that cannot allocate
 * device memory (code inside another framework's memory pool, host callbacks that
 * must not allocate, processes whose device memory belongs to a pool they do not
 * control).  The pages have no counterpart: their quantiser runs through PyTorch and
 * may allocate freely.
 * The scratch lives in a fixed file-scope device array for tensors of up to
 * nf4ls_quantize_noalloc_max_elems() weights (2^28, 16 MiB of device memory held by
 * every GPU that loads the library until the process exits).  Larger n returns
 * NF4LS_INVALID_ARG.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make it before any stream capture.  The first call in a
 * new CUDA context on that device (after a device reset, or under a context the
 * caller created) looks it up again, since an address is valid only in the context
 * it came from.  All calls share the
 * array, so calls that overlap on the GPU race; serialise them on one stream.  No
 * part of the array needs to start at zero.  Allocates nothing; results are the same
 * bytes nf4_quantize_tensor produces. */
size_t nf4ls_quantize_noalloc_max_elems(void);
int nf4_quantize_tensor_noalloc(const void* w_dev, size_t n, uint8_t* packed_dev, uint8_t* q8_dev,
                                float* nested_dev, float* offset_dev, nf4ls_stream stream);

/* ------------------------------------------------------------------ layer shards
 * A shard is one decoder layer as one contiguous byte range, the unit that streams
 * ([gate] §2.1: offline per-layer shards; [review]: the cache key carries the
 * quantisation method and the source checkpoint fingerprint).  Layout:
 *   [0, 256)    nf4ls_shard_header
 *   [256, 832)  nf4ls_tensor_desc[9]  (q, k, v, o, gate, up, down, norm_in, norm_post)
 *   then each region 256-byte aligned: packed, q8, nested, offset of the seven
 *   linears, then the two bf16 RMSNorm weights [H] copied verbatim.
 * Offsets in the descriptors are relative to the shard start, so a shard is
 * position independent: it may live in the pinned store, in any pool slot or
 * resident in HBM, and the kernels read it the same way. */
#define NF4LS_SHARD_MAGIC   0x5334464Eu /* "NF4S" little-endian */
#define NF4LS_SHARD_VERSION 1u
#define NF4LS_METHOD_NF4_DQ 1u

typedef struct {
    uint32_t magic, version, method, blocksize;      /* blocksize = 64            */
    uint32_t nested_blocksize, n_tensors;            /* 256, 9                    */
    uint32_t hidden, inter, n_q, n_kv, head_dim, pad0;
    uint64_t codebook_hash, fingerprint, total_bytes;
    uint64_t quantized_bytes;                        /* sum of the identity bytes */
    uint8_t reserved[256 - 80];
} nf4ls_shard_header;

typedef struct {
    uint32_t kind, format;                           /* format 1 = NF4-DQ, 2 = bf16 */
    uint64_t rows, cols;
    uint64_t off_packed, off_q8, off_nested, off_offset;  /* bf16: off_packed = data */
    uint64_t pad;
} nf4ls_tensor_desc;

/* Bytes of one shard for cfg (header, descriptors, aligned regions). */
size_t nf4ls_shard_bytes(const nf4ls_layer_cfg* cfg);
/* Sum of the per-tensor identity bytes (n/2 + n/64 + 4*ceil(n/16384) + 4) of the seven linears. */
size_t nf4ls_shard_quantized_bytes(const nf4ls_layer_cfg* cfg);
size_t nf4ls_shard_scratch_bytes(const nf4ls_layer_cfg* cfg);

/* Quantises one decoder layer into a shard ([gate] §2.1, one tensor at a time on
 * the GPU).  weights_dev[9]: bf16 device pointers in shard order (the seven
 * linears [out, in], then norm_in [H], norm_post [H]).  shard_dev receives
 * nf4ls_shard_bytes(cfg) bytes (cap must be at least that); *used gets the count.
 * fingerprint identifies the source checkpoint and is stored in the header. */
int nf4_quantize_shard(const nf4ls_layer_cfg* cfg, const void* const* weights_dev,
                       uint64_t fingerprint, void* shard_dev, size_t cap, size_t* used,
                       void* scratch_dev, size_t scratch_bytes, nf4ls_stream stream);

/* Host-side check of a shard header (a copy in host memory): magic, version,
 * method, code-table hash and, when expected_fingerprint != 0, the fingerprint. */
int nf4ls_shard_check(const void* header_host, const nf4ls_layer_cfg* cfg,
                      uint64_t expected_fingerprint);

/* ------------------------------------------------------------------ layer calls
 * LoRA adapter on q_proj and v_proj (resident in HBM, fp32 masters):
 *   A_q [r, H], B_q [n_q*d, r], A_v [r, H], B_v [n_kv*d, r]; scale = alpha / r.
 * The kernels cast A and B to bf16 for the products, as the pages' bf16 compute does. */
typedef struct {
    const float* A_q;
    const float* B_q;
    const float* A_v;
    const float* B_v;
} nf4ls_lora;

typedef struct {
    float* dA_q;
    float* dB_q;
    float* dA_v;
    float* dB_v;
} nf4ls_lora_grads;

/* Workspace of layer_forward / layer_backward for cfg (cfg->batch * cfg->seq tokens). */
size_t nf4ls_workspace_bytes(const nf4ls_layer_cfg* cfg);

/* One decoder layer forward ([gate] §2.1: the HF Llama layer body):
 *   h1 = rmsnorm(x) w_in; q,k,v = h1 W^T (+ s (h1 A^T) B^T on q and v); RoPE on q,k;
 *   o = causal GQA attention; h = x + o Wo^T; h2 = rmsnorm(h) w_post;
 *   a = silu(h2 Wg^T) * (h2 Wu^T); y = h + a Wd^T.
 * shard_dev: the layer's shard (pool slot or resident).  x_dev, y_dev: bf16 [M, H].
 * lora may be NULL: the adapter is off (the same frozen base serves as reference). */
int layer_forward(const nf4ls_layer_cfg* cfg, const void* shard_dev, const nf4ls_lora* lora,
                  const void* x_dev, void* y_dev, void* ws_dev, size_t ws_bytes,
                  nf4ls_stream stream);

/* Checkpoint recompute + backward of one layer ([review] mechanism section: the
 * layer is read twice per step and dL/dx = W^T dL/dy flows through the frozen base;
 * [gate] §4.4: no dL/dW).  x_saved_dev: the layer input saved by the forward;
 * dy_dev: dL/dy bf16 [M, H]; dx_dev: dL/dx bf16 [M, H] (may alias dy_dev).
 * grads (fp32, written, not accumulated) may be NULL when lora is NULL.
 * Deterministic: no atomics, fixed reduction orders. */
int layer_backward(const nf4ls_layer_cfg* cfg, const void* shard_dev, const nf4ls_lora* lora,
                   const void* x_saved_dev, const void* dy_dev, void* dx_dev,
                   const nf4ls_lora_grads* grads, void* ws_dev, size_t ws_bytes,
                   nf4ls_stream stream);

/* GEMM path selection (process-wide; default 0):
 *   0 = NF4 decode inside the tcgen05 GEMM mainloop;
 *   1 = dequantise the layer to bf16 in the workspace, then the dense tcgen05 GEMM.
 * Both give bit-identical results (same decoded values, same MMA order). */
int nf4ls_set_gemm_path(int path);

/* CTA-pair GEMMs (process-wide; default 1): products with more than 256 tokens run
 * on clusters of two CTAs sharing one 2-SM tcgen05 MMA (512 tokens x 256 features per
 * pair); 0 keeps one CTA per 256 x 256 tile.  For testing and comparison. */
int nf4ls_set_gemm_pair(int on);

/* Token height of the CTA-pair tiles (process-wide; default 0): 0 = choose per launch
 * between 512 and 256 by their tile-times; 1 = always 512; 2 = always 256
 * (128 per CTA, one accumulator); 3 = 512-token tiles for the whole waves and the tiles
 * of the last, partial wave as 256-token tiles in a second launch (where every
 * 512-token tile is two 256-token tiles, else as 1).  Results do not depend on it (same
 * reduction order per output).  For testing and comparison. */
int nf4ls_set_gemm_half(int mode);

/* Attention forward (process-wide; default 1): 1 = the tcgen05 kernel (scores and
 * output accumulated in TMEM) where head_dim is 128 and seq a multiple of 128 up to
 * 512, the mma.sync kernel elsewhere; 0 = always the mma.sync kernel.  The two agree
 * up to fp32 summation order.  For testing and comparison. */
int nf4ls_set_attention_path(int tc);

/* ------------------------------------------------------------------ streaming pool
 * [review] mechanism section: the frozen base lives in pinned host memory; 2-8
 * preallocated HBM buffers (double by default) are filled on a dedicated CUDA
 * stream, prefetching layer i+1 in the forward and i-1 in the backward so the copy
 * overlaps compute.  [review] bug history (#331): a buffer may be overwritten only
 * after every kernel that reads it has finished; here the copy into a slot waits on
 * an event recorded on the compute stream when the slot was released.
 *
 * pinned_host: the pinned store; layer_off[i], layer_bytes[i]: byte range of layer
 * i's shard in it.  slots_dev: depth * slot_bytes bytes of device memory (caller's),
 * slot_bytes >= every layer_bytes[i] and a multiple of 256.  depth in [2, 8].
 * Slots are reused least-recently-released first; a layer still in a slot is not
 * copied again (so the last layers of the forward are reused by the backward). */
typedef struct nf4ls_pool nf4ls_pool;

typedef struct {
    uint64_t bytes_copied;   /* host-to-device bytes issued          */
    uint64_t copies;         /* layer copies issued                  */
    uint64_t hits;           /* acquisitions served without a copy   */
    uint64_t acquisitions;
    uint64_t peer_bytes;     /* bytes received from other GPUs (shared fetch) */
} nf4ls_pool_stats;

int nf4ls_pool_create(const void* pinned_host, const size_t* layer_off, const size_t* layer_bytes,
                      int n_layers, int depth, void* slots_dev, size_t slot_bytes, nf4ls_pool** out);
/* Issues the copy of layer into a free slot on the pool's copy stream if it is not
 * already resident (non-blocking).  NF4LS_BUFFER_BUSY if every slot is acquired. */
int nf4ls_pool_prefetch(nf4ls_pool* pool, int layer);
/* Acquires layer for the compute stream: issues its copy if needed, makes `compute`
 * wait on the copy's event, and returns the slot's device address.  The slot stays
 * acquired until nf4ls_pool_release. */
int stream_prefetch(nf4ls_pool* pool, int layer, nf4ls_stream compute, const void** slot_dev);
/* Records on `compute` the event that frees layer's slot once the kernels enqueued
 * so far (its last readers) have finished. */
int nf4ls_pool_release(nf4ls_pool* pool, int layer, nf4ls_stream compute);
/* Host wait, bounded by timeout_ms, for layer's copy to finish.  NF4LS_TIMEOUT. */
int nf4ls_wait(nf4ls_pool* pool, int layer, int timeout_ms);
/* Debug: fill every released slot with 0xFF before its next copy, so that any read
 * of a released slot (an aliasing bug) corrupts results grossly and reproducibly. */
int nf4ls_pool_set_poison(nf4ls_pool* pool, int on);
int nf4ls_pool_get_stats(nf4ls_pool* pool, nf4ls_pool_stats* out);
int nf4ls_pool_synchronize(nf4ls_pool* pool);
int nf4ls_pool_destroy(nf4ls_pool* pool);

/* ------------------------------------------------------------------ layer-sharded fetch
 * Data-parallel ranks stream the same shards; since the step is bound by each GPU's
 * host-to-device link, ranks can split the fetch: rank r's pool copies from its host
 * store only the layers it owns (layer % world == r) and every slot fill becomes an
 * NCCL broadcast of the layer from its owner's slot into the other ranks' slots, over
 * NVLink, on the pool's copy stream.  The bytes in every slot are those a private
 * copy would have brought, so results are unchanged.  Every rank's pool must see the
 * same sequence of prefetch / stream_prefetch / release calls (a data-parallel step
 * does), so that the broadcasts pair up; a pool with a file store cannot be shared.
 * nf4ls_nccl_unique_id: rank 0 makes the id, the caller distributes it;
 * nf4ls_pool_share: called by every rank at the same time (NCCL communicator set-up). */
int nf4ls_nccl_unique_id(uint8_t id_out[128]);
int nf4ls_pool_share(nf4ls_pool* pool, int rank, int world, const uint8_t id[128]);

/* ------------------------------------------------------------------ slot plan (host only)
 * The slot decisions behind every pool call, with no device work, so that they can be
 * checked without a GPU (for instance on several CPU ranks, for the sharded fetch):
 * the pool takes each of its decisions through this same plan object.  A plan has the
 * pool's depth and layer count; nf4ls_plan_share switches it to the sharded fetch
 * (before it holds a layer, as nf4ls_pool_share).  nf4ls_plan_prefetch,
 * nf4ls_plan_acquire and nf4ls_plan_release mirror nf4ls_pool_prefetch,
 * stream_prefetch and nf4ls_pool_release, return the same statuses
 * (NF4LS_BUFFER_BUSY when every slot is acquired or filled and not yet acquired, or
 * when the layer is already acquired; the plan is then unchanged) and fill `out`
 * (may be NULL) with what the pool does for that call. */
typedef struct nf4ls_plan nf4ls_plan;

typedef struct {
    int32_t slot;           /* the slot that serves the layer                            */
    int32_t hit;            /* 1: the layer already sat in that slot, nothing is copied  */
    int32_t fill;           /* 1: this call fills the slot                               */
    int32_t after_release;  /* 1: the fill waits for the slot's previous release event   */
    int32_t owner;          /* the rank that reads the layer from its host store         */
    int32_t host_read;      /* 1: this rank copies it from its own store                 */
    int32_t broadcast;      /* 1: shared pool: the fill is a broadcast from the owner    */
} nf4ls_plan_step;

int nf4ls_plan_create(int n_layers, int depth, nf4ls_plan** out);
int nf4ls_plan_share(nf4ls_plan* plan, int rank, int world);
int nf4ls_plan_prefetch(nf4ls_plan* plan, int layer, nf4ls_plan_step* out);
int nf4ls_plan_acquire(nf4ls_plan* plan, int layer, nf4ls_plan_step* out);
int nf4ls_plan_release(nf4ls_plan* plan, int layer);
int nf4ls_plan_destroy(nf4ls_plan* plan);

/* The pool calls one pass of nf4ls_forward_backward makes (dir +1: the forward over
 * layers 0..n-1; dir -1: the backward over n-1..0), in order: op 0 = acquire
 * (stream_prefetch), 1 = prefetch (nf4ls_pool_prefetch; on NF4LS_BUFFER_BUSY the step
 * skips the remaining prefetches for that layer), 2 = run the layer, 3 = release.
 * ops[i], layers[i] for i < *n_out; NF4LS_INVALID_ARG (with *n_out set) when cap is
 * too small. */
int nf4ls_step_pass_ops(int n_layers, int dir, int32_t* ops, int32_t* layers, int cap, int32_t* n_out);

/* ------------------------------------------------------------------ disk stream source
 * [review] mechanism section: the frozen base lives in (pinned) host memory and falls
 * back to an NVMe disk when memory is short; SATA and spinning disks are refused
 * outright; the config key stream_source: auto takes memory when the store fits and
 * NVMe otherwise.
 *
 * nf4ls_disk_probe: classifies the device under `path` (sysfs: block device or not,
 * NVMe, rotational) and times a sequential read of up to probe_bytes of the file
 * (O_DIRECT when the file system allows it, so the page cache does not answer).
 * nf4ls_disk_accept: NF4LS_OK for a non-rotational device that is NVMe or not a block
 * device at all (memory-backed) and reads at >= min_gbs; NF4LS_SOURCE_REFUSED
 * otherwise (the message says why).
 * nf4ls_choose_source: *use_disk = 0 when store_bytes + reserve_bytes fit in the
 * host's available memory (MemAvailable), else 1. */
typedef struct {
    double read_gbs;        /* measured sequential read, GB/s (1e9 B/s)        */
    int32_t block_device;   /* 1: the file sits on a block device              */
    int32_t nvme;           /* 1: ... and that device is NVMe                  */
    int32_t rotational;     /* 1: ... and it is a spinning disk                */
    int32_t direct_io;      /* 1: the probe read with O_DIRECT                 */
} nf4ls_disk_info;

int nf4ls_disk_probe(const char* path, size_t probe_bytes, nf4ls_disk_info* out);
int nf4ls_disk_accept(const nf4ls_disk_info* info, double min_gbs);
int nf4ls_choose_source(size_t store_bytes, size_t reserve_bytes, int32_t* use_disk);

/* A pool whose store is a file: layer i is bytes [layer_off[i], + layer_bytes[i]) of
 * `path` (layer_off[i] a multiple of 4096, so reads can bypass the page cache).  A
 * reader thread reads each requested layer into one of two pinned staging buffers
 * (staging_host: caller's pinned memory, 4096-byte aligned, >= 2 x the largest layer
 * rounded up to 4096; nf4ls_pool_file_staging_bytes) and issues its host-to-device
 * copy on the pool's copy stream; stream_prefetch then returns once that copy is
 * enqueued (a host wait of at most 60 s, NF4LS_TIMEOUT after).  Every other pool call
 * behaves as for a pinned store, and the bytes that reach a slot are the same. */
size_t nf4ls_pool_file_staging_bytes(const size_t* layer_bytes, int n_layers);
int nf4ls_pool_create_file(const char* path, const size_t* layer_off, const size_t* layer_bytes, int n_layers,
                           int depth, void* slots_dev, size_t slot_bytes, void* staging_host, size_t staging_bytes,
                           nf4ls_pool** out);

/* ------------------------------------------------------------------ model step
 * One SFT step of the whole stack ([review]: embeddings and lm_head stay resident
 * and unquantised; [gate] §4.4: lm_head outside the checkpointed layers):
 * embedding gather -> n_layers x layer_forward (streamed or resident, saving each
 * layer input) -> final RMSNorm -> logits = h lm_head^T -> causal-LM cross-entropy
 * (logits[t] vs ids[t+1], mean over batch*(seq-1)) -> dh through lm_head -> final
 * norm backward -> layer_backward in reverse order -> AdamW on every LoRA tensor.
 *
 * LoRA parameters, gradients and AdamW moments are fp32 arrays laid out per layer
 * with stride nf4ls_lora_stride(cfg) floats: [A_q | B_q | A_v | B_v]. */
typedef struct {
    nf4ls_layer_cfg layer;
    int32_t n_layers;
    int32_t vocab;
    int32_t tied;            /* 1: lm_head is the embedding table      */
    float lr, beta1, beta2, adam_eps, weight_decay;
    /* 0: embedding and lm_head resident in HBM (embed_dev, lm_head_dev).
     * > 0: the streamed head ([gate] §4.3 lists streaming the unquantised embedding and
     * lm_head "as a large layer" as the next step): the output matrix (lm_head, or the
     * embedding when tied) is read in vocab chunks of head_chunk_rows rows (a multiple
     * of 64) through head_pool, and the embedding rows of the batch are gathered from
     * embed_host when embed_dev is NULL.  The loss and dL/dh come from one pass over
     * the chunks: per row a running max and sum of exp, and the sum of
     * exp(logit - max) * lm_head row rescaled whenever the max grows, so the [M, V]
     * logits are never stored. */
    int32_t head_chunk_rows;
} nf4ls_model_cfg;

typedef struct {
    const void* embed_dev;        /* bf16 [V, H]                        */
    const void* lm_head_dev;      /* bf16 [V, H]; ignored when tied     */
    const void* norm_final_dev;   /* bf16 [H]                           */
    float* lora_dev;              /* fp32 [n_layers * stride]           */
    float* grads_dev;             /* fp32 [n_layers * stride]           */
    float* adam_m_dev;            /* fp32 [n_layers * stride]           */
    float* adam_v_dev;            /* fp32 [n_layers * stride]           */
    nf4ls_pool* pool;             /* streamed shards, or NULL ...       */
    const void* const* shards_dev;/* ... resident shard pointers        */
    void* ws_dev;
    size_t ws_bytes;
    /* streamed head only (head_chunk_rows > 0), else NULL: */
    nf4ls_pool* head_pool;        /* layer i = bf16 rows [i c, min(V, (i+1) c)) x H of
                                     the output matrix, c = head_chunk_rows            */
    const void* embed_host;       /* bf16 [V, H] in pinned host memory the device can
                                     read (mapped), used when embed_dev is NULL         */
} nf4ls_model;

size_t nf4ls_lora_stride(const nf4ls_layer_cfg* cfg);
size_t nf4ls_model_workspace_bytes(const nf4ls_model_cfg* cfg);
/* ids_dev: int32 [batch, seq].  step counts from 1 (AdamW bias correction).
 * loss_dev: fp32 [1] receives the mean loss.  lora_on = 0 runs the frozen base only
 * (no gradients, no update): the adapter-off reference pass of DPO/KTO. */
int nf4ls_train_step(const nf4ls_model_cfg* cfg, const nf4ls_model* model, const int32_t* ids_dev,
                     int32_t step, float* loss_dev, nf4ls_stream stream);
int nf4ls_forward_loss(const nf4ls_model_cfg* cfg, const nf4ls_model* model, const int32_t* ids_dev,
                       int32_t lora_on, float* loss_dev, nf4ls_stream stream);
/* The two halves of nf4ls_train_step, for data parallelism: forward + backward
 * writes the LoRA gradients (fp32, per-layer stride) into grads_dev; the caller may
 * all-reduce them across ranks and then apply nf4ls_adamw_step. */
int nf4ls_forward_backward(const nf4ls_model_cfg* cfg, const nf4ls_model* model, const int32_t* ids_dev,
                           float* loss_dev, nf4ls_stream stream);
int nf4ls_adamw_step(const nf4ls_model_cfg* cfg, const nf4ls_model* model, int32_t step, nf4ls_stream stream);

/* ------------------------------------------------------------------ adapter checkpoint
 * Save / resume of the trainable state: the LoRA parameters and both AdamW moments
 * (model->lora_dev, adam_m_dev, adam_v_dev, n_layers * nf4ls_lora_stride floats
 * each) and the number of AdamW steps taken.  [gate] §3.2: a release's adapters
 * were trained correctly but reloaded as empty, unseen because no test saved and
 * reloaded one; loading here either restores the exact bytes or fails.
 *
 * File: a 64-byte header (magic NF4LS_ADAPTER_MAGIC, version, H, I, n_q, n_kv,
 * head_dim, lora_r, n_layers, lora_alpha, step, floats per array, FNV-1a 64
 * checksum over the header with that field zeroed and then the arrays) then the
 * three fp32 arrays, little-endian, in the device layout.  nf4ls_adapter_file_bytes
 * gives its size (0 for a NULL or empty config).
 *
 * nf4ls_adapter_save: copies the three arrays to the host on `stream` (ordered after
 * the steps already queued there), writes path + ".tmp", fsyncs it, renames it to
 * path and fsyncs the directory, so an interrupted save leaves an older file at
 * path intact and a completed one survives a crash.  step >= 0 is stored as given:
 * pass the count of AdamW steps applied so far.  NF4LS_IO on a failed open / write /
 * rename / directory flush (the temporary file is removed).
 *
 * nf4ls_adapter_load: reads and checks the whole file first; NF4LS_INVALID_ARG for a
 * wrong magic or version (files of version 1, whose checksum left the header out,
 * are refused), NF4LS_SHAPE when H, I, heads, head_dim, lora_r, lora_alpha,
 * n_layers or the array size differ from cfg (batch and seq may differ), NF4LS_IO
 * for a short, over-long or checksum-failing file.  Only then are the three device
 * arrays overwritten (on `stream`, synchronised before return) and *step set; on any
 * failure the model is left as it was.  The next nf4ls_train_step / adamw_step of
 * the resumed run passes *step + 1.  The gradient buffer is not saved: every step
 * rewrites it. */
#define NF4LS_ADAPTER_MAGIC   0x41344E46u /* "FN4A" little-endian */
#define NF4LS_ADAPTER_VERSION 2u
size_t nf4ls_adapter_file_bytes(const nf4ls_model_cfg* cfg);
int nf4ls_adapter_save(const char* path, const nf4ls_model_cfg* cfg, const nf4ls_model* model, int32_t step,
                       nf4ls_stream stream);
int nf4ls_adapter_load(const char* path, const nf4ls_model_cfg* cfg, const nf4ls_model* model, int32_t* step,
                       nf4ls_stream stream);

/* Loss of the single-layer workloads: loss = mean(out^2) over n values and
 * dout = bf16(2 out / n).  partial_dev: n_partial (1..4096) floats of scratch. */
int nf4ls_mse_loss(const void* out_dev, size_t n, void* dout_dev, float* loss_dev, float* partial_dev,
                   int n_partial, nf4ls_stream stream);

/* ------------------------------------------------------------------ building blocks
 * Exported so that tests can check each kernel on its own; layer_forward and
 * layer_backward are built from these. */

/* Dense bf16 GEMM on the tcgen05 tensor cores: out[M, N] = A[M, K] B^T where
 * B is [N, K] (b_trans = 0) or B is stored [K, N] (b_trans = 1, i.e. out = A B).
 * K % 64 == 0; fp32 accumulation; out bf16 with leading dimension ldo. */
int nf4ls_gemm_bf16(const void* A_dev, const void* B_dev, void* out_dev, int M, int N, int K,
                    int b_trans, int ldo, nf4ls_stream stream);

/* The same tcgen05 GEMM with one NF4 tensor W [rows, cols] decoded inside the
 * mainloop: dgrad = 0: out[M, rows] = A[M, cols] W^T; dgrad = 1: out[M, cols] =
 * A[M, rows] W.  rows % 64 == 0, cols % 64 == 0. */
int nf4ls_gemm_nf4(const void* A_dev, int lda, int M, const uint8_t* packed_dev, const uint8_t* q8_dev,
                   const float* nested_dev, const float* offset_dev, int rows, int cols, int dgrad,
                   void* out_dev, int ldo, nf4ls_stream stream);

/* Causal GQA attention forward: q [M, n_q*d], k/v [M, n_kv*d] (row stride ld_q/ld_kv
 * elements) -> o [M, n_q*d] bf16 and lse fp32 [batch, n_q, seq]. */
int nf4ls_attention_fwd(const nf4ls_layer_cfg* cfg, const void* q_dev, const void* k_dev,
                        const void* v_dev, int ld_q, int ld_kv, void* o_dev, float* lse_dev,
                        nf4ls_stream stream);

/* Its backward: from q, k, v (as above), o and do [M, n_q*d] (row stride n_q*d), lse
 * [batch, n_q, seq] of the forward -> dq [M, n_q*d], dk, dv [M, n_kv*d] (bf16, row
 * strides n_q*d and n_kv*d) and delta = rowsum(do * o) fp32 [batch, n_q, seq] (a
 * by-product, written).  dq, dk, dv are the gradients with respect to the forward's
 * q, k, v (before any RoPE transpose). */
int nf4ls_attention_bwd(const nf4ls_layer_cfg* cfg, const void* q_dev, const void* k_dev,
                        const void* v_dev, int ld_q, int ld_kv, const void* o_dev, const void* do_dev,
                        const float* lse_dev, float* delta_dev, void* dq_dev, void* dk_dev, void* dv_dev,
                        nf4ls_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* NF4LS_H */
