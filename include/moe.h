/*
 * moe.h -- C ABI of libmoe: the per-token Mixture-of-Experts layer of a
 * "streaming experts" decoder, on NVIDIA B200 (sm_100a).
 *
 * What the layer computes (the pages describe the Flash-MoE engine that runs
 * Qwen3.5-397B-A17B with experts streamed from SSD):
 *   1. router: logits = x . Wr^T + bias; the top K of E experts per token,
 *      weights = softmax over E renormalised over the K chosen
 *      ("Streaming experts: как запустить триллионную модель на MacBook"
 *      (toolarium.ru), section "Mixture of Experts и почему SSD достаточно":
 *      4 of 512 experts per token; "Flash-MoE: ラップトップでの397Bパラメータ
 *      モデルの実行" (hakusoku.com), section "パイプライン概要": CPU
 *      softmax/top-K after the GPU router projection);
 *   2. for each chosen expert, a SwiGLU FFN whose weights are 4- or 2-bit
 *      group-affine codes, dequantised as q*scale + bias and multiplied in the
 *      fused form fma(q, scale*x, bias*x) (toolarium, section "Оптимизации,
 *      которые сработали"; hakusoku, section "主要技術": FMA dequant kernel,
 *      4/2-bit dequant matvec, SwiGLU);
 *   3. a shared expert (bf16 SwiGLU FFN, weight 1) (hakusoku, section
 *      "モデルアーキテクチャ": K=4 plus a shared expert);
 *   4. combine + residual + RMSNorm in one kernel (toolarium, section
 *      "Оптимизации, которые сработали"; hakusoku, section "主要技術").
 *
 * Conventions for every call:
 *   - Pointers are owned by the caller.  Device pointers are CUDA global
 *     memory on the current device; host pointers are ordinary host memory
 *     (pinned where stated).  The library allocates no device memory,
 *     except the slots of an expert-streaming cache (moe_stream_create).
 *   - Device calls are asynchronous on the given stream and do not
 *     synchronise unless stated.  Inputs are never modified.
 *   - Every call returns a moe_status.  On MOE_OK all outputs are fully
 *     written (once the stream reaches them); on an error they are
 *     unspecified.  moe_last_error() gives a message for the last failing
 *     call on the calling host thread.
 *   - bf16 tensors are passed as 16-bit patterns (void*), row-major.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad index */
  MOE_ERR_UNSUPPORTED = 2, /* bits not 2/4, group not 64, H or I not a multiple of 64, K > E, T too large for the path */
  MOE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the size query says */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call failed (message has the CUDA error) */
  MOE_ERR_OOM = 5,         /* a device or pinned-host allocation failed */
  MOE_ERR_TIMEOUT = 6,     /* a bounded device-side wait expired (see moe_device_error) */
  MOE_ERR_IO = 7,          /* the expert-streaming tier could not copy from its host store */
  MOE_ERR_DEVICE = 8       /* a device-side check failed (misaligned expert pointer, bad expert id) */
} moe_status;

/* Layer shape.  hidden H, inter I (expert intermediate size), n_experts E,
 * top_k K, bits b (4 or 2), group G (64), eps of the RMSNorm (1e-6 in the
 * synthetic workloads), has_shared (1 = a bf16 shared expert of the same I). */
typedef struct {
  int hidden, inter, n_experts, top_k, bits, group;
  float eps;
  int has_shared;
} moe_config;

/* Thread-local message for the last failing call ("" if none). */
const char* moe_last_error(void);

/* ------------------------------------------------------------------------
 * Packed expert format (this library's; the pages fix only the size, ~6.75 MB
 * per 4-bit expert at H=4096, toolarium, section "Flash-MoE: чистый C, Metal и
 * никакого Python").  One blob per expert, six sections each starting on a
 * 256-byte boundary:
 *   0 gate codes [I][H*b/8]   1 up codes [I][H*b/8]   2 down codes [H][I*b/8]
 *   3 gate scales [I][H/G]    4 up scales [I][H/G]    5 down scales [H][I/G]
 * Codes come in blocks of 8 rows x 64 columns (one group of 8 rows), ordered
 * by row block, then column group; a block is 64*b bytes.  Inside a block,
 * "lane" l = 4*(row % 8) + t (t = 0..3) owns 2*b consecutive bytes
 * (little-endian 32-bit words) holding, for each 16-column step s = 0..3 of
 * the group, the columns 16s + 2t + e ("first") and 16s + 8 + 2t + e
 * ("second"), e = 0, 1 -- the codes a tensor-core B fragment of an m16n8k16
 * step takes for that lane:
 *   4-bit: word s/2; code at nibble 2(s%2) + 4e (first) or 2(s%2) + 1 + 4e
 *          (second);
 *   2-bit: one word; code at 2-bit slot 2s + 8e (first) or 2s + 1 + 8e
 *          (second).
 * Scale words are stored [row block][group][row % 8].  A run of whole row
 * blocks is therefore one contiguous byte range in both sections.
 * Scale word (uint32): bf16 scale s in bits 0..15, bf16 bias beta in bits
 * 16..31; weight = q*s + beta.  Groups run along the input (reduction) dim.
 * Quantiser (round-to-nearest affine, single precision):
 *   s = bf16_rne((max-min)/(2^b-1)), beta = bf16_rne(min),
 *   q = clamp(rint((w - beta)/s), 0, 2^b-1), q = 0 when s == 0.
 * Blob size: moe_packed_expert_bytes (7,077,888 B at H=4096, I=1024, 4-bit;
 * 3,932,160 B at 2-bit).  Blobs handed to the device calls must start on a
 * 256-byte boundary.
 * ------------------------------------------------------------------------ */

/* Bytes of one packed expert; 0 if cfg is unsupported. */
size_t moe_packed_expert_bytes(const moe_config* cfg);

/* Byte offsets of the six sections inside a blob. */
moe_status moe_packed_layout(const moe_config* cfg, size_t offsets[6]);

/* Host packer (the pages' offline repacking scripts for 4-bit and 2-bit
 * experts, hakusoku, section "プロジェクト構成").  w_gate, w_up: fp32
 * [*][I][H]; w_down: fp32 [*][H][I] (host).  Packs experts e_begin ..
 * e_begin+e_count-1 of those arrays into out (host, e_count consecutive blobs
 * of moe_packed_expert_bytes each; out_bytes must be at least that).
 * Inputs must be finite.  Synchronous, multi-threaded over experts. */
moe_status moe_pack_experts(const moe_config* cfg, const float* w_gate, const float* w_up,
                            const float* w_down, int e_begin, int e_count, void* out,
                            size_t out_bytes);

/* Device packer: the same format and bit-identical output as
 * moe_pack_experts, computed on the GPU.  w_gate, w_up: fp32 [e_count][I][H],
 * w_down: fp32 [e_count][H][I] (device); out: device, e_count blobs. */
moe_status moe_pack_experts_device(const moe_config* cfg, const float* w_gate,
                                   const float* w_up, const float* w_down, int e_count,
                                   void* out, size_t out_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Router (toolarium, section "Mixture of Experts и почему SSD достаточно";
 * hakusoku, section "パイプライン概要").
 *   logits[t][e] = sum_h x[t][h]*Wr[e][h] (fp32 accumulation) + bias[e]
 *   idx[t][0..K-1]: the K largest logits, descending, ties to the lower index
 *     (a NaN logit ranks as -inf)
 *   w[t][k] = exp(l_k - l_max) / sum_j exp(l_j - l_max) over the K chosen
 *     (= softmax over E renormalised over the K).
 * x_bf16 [T][H], wr_bf16 [E][H], bias fp32 [E] or NULL, idx int32 [T][K],
 * w fp32 [T][K], logits_out fp32 [T][E] or NULL: all device.  If logits_out
 * is NULL the logits go to workspace (moe_router_workspace_bytes). */
size_t moe_router_workspace_bytes(const moe_config* cfg, int T);
moe_status moe_router_topk(const moe_config* cfg, const void* x_bf16, const void* wr_bf16,
                           const float* bias, int T, int32_t* idx, float* w,
                           float* logits_out, void* workspace, size_t ws_bytes,
                           cudaStream_t stream);

/* Top-K and weights from given fp32 logits [T][E] (device), same rules. */
moe_status moe_topk_from_logits(const moe_config* cfg, const float* logits, int T,
                                int32_t* idx, float* w, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Whole layer.
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* const* expert_ptr; /* device array [E] of device pointers, one packed blob per expert (256-B aligned) */
  const void* router_w;          /* bf16 [E][H] */
  const float* router_bias;      /* fp32 [E] or NULL */
  const void* shared_gate;       /* bf16 [I][H]; ignored when has_shared == 0 */
  const void* shared_up;         /* bf16 [I][H] */
  const void* shared_down;       /* bf16 [H][I] */
  const void* gamma;             /* bf16 [H], RMSNorm weight */
  /* Optional forms of the shared expert (both NULL: the bf16 FFN above with
   * weight 1).  The pages name a shared expert next to the K routed ones and
   * compute it in the GPU command with the router (hakusoku
   * "モデルアーキテクチャ", "パイプライン概要") without printing its form. */
  const void* shared_out_gate;   /* bf16 [H] or NULL: the shared output is scaled by
                                    sigmoid(x . shared_out_gate) (fp32 dot) */
  const void* shared_packed;     /* device blob in the routed experts' packed format
                                    (moe_pack_experts, 256-B aligned) or NULL: when set it
                                    replaces shared_gate/up/down, which may then be NULL */
} moe_layer_weights;

/* Workspace for moe_layer_forward with T tokens (device memory, 256-B
 * aligned).  It must be zero-filled once before its first use
 * (moe_workspace_init); the layer leaves it ready for the next call.  One
 * workspace serves one call at a time: calls that overlap on the GPU must use
 * different workspaces. */
size_t moe_layer_workspace_bytes(const moe_config* cfg, int T);
moe_status moe_workspace_init(void* workspace, size_t ws_bytes, cudaStream_t stream);

/* One MoE layer for T tokens (device pointers):
 *   h_out[t]  = residual[t] + sum_k w[t][k] * expert_{idx[t][k]}(x[t]) + shared(x[t])
 *   y_norm[t] = h_out[t] / sqrt(mean(h_out[t]^2) + eps) * gamma
 * expert_e(x) = Wd_e (silu(Wg_e x) * (Wu_e x)) with dequantised weights.
 * x_bf16, residual_bf16 [T][H]; h_out_bf16, y_norm_bf16 [T][H] (y_norm is
 * computed from the fp32 sum, before h_out is rounded to bf16); idx_out
 * int32 [T][K] and w_out fp32 [T][K] may be NULL.  T == 0 is a no-op.
 * For T < 32, one launch of the fused kernel takes C =
 * moe_layer_tokens_per_launch(cfg) tokens and a larger T runs as successive
 * launches of C tokens on the stream (each token's result depends on that
 * token only; each launch reads the experts its tokens chose).  From T = 32
 * the call takes the batched path (moe_layer_forward_batched) when the shape
 * allows it.  moe_layer_workspace_bytes covers whichever path runs.
 * A bounded device wait that expires leaves MOE_ERR_TIMEOUT in the
 * workspace (moe_device_error). */
moe_status moe_layer_forward(const moe_config* cfg, const moe_layer_weights* wts,
                             const void* x_bf16, const void* residual_bf16, int T,
                             void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out,
                             float* w_out, void* workspace, size_t ws_bytes,
                             cudaStream_t stream);

/* The batched form of the layer (same arguments and results as
 * moe_layer_forward), for batches where several tokens share an expert:
 * router logits as a GEMM, top-K, the T*K (token, expert) pairs grouped by
 * expert, then per chosen expert and chunk of up to 128 of its tokens a
 * gate/up GEMM and a down GEMM on the tensor cores with the expert's packed
 * weights dequantised once per chunk (weights and activations of the routed
 * experts enter as fp16, accumulation in fp32), the shared expert as bf16
 * GEMMs (its intermediate as bf16 hi + lo), and one combine + residual +
 * RMSNorm pass.  Workspace: moe_layer_batched_workspace_bytes (grows with T:
 * about T * K * (2 I + 4 H) bytes).  n_experts <= 2048.  Expert pointers are
 * checked (non-null, 256-byte aligned) before any is read; a bad one leaves
 * MOE_ERR_DEVICE in the workspace (moe_device_error) and the outputs
X
size_t moe_layer_batched_workspace_bytes(const moe_config* cfg, int T);
moe_status moe_layer_forward_batched(const moe_config* cfg, const moe_layer_weights* wts,
                                     const void* x_bf16, const void* residual_bf16, int T,
                                     void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out,
                                     float* w_out, void* workspace, size_t ws_bytes,
                                     cudaStream_t stream);

/* The layer through the fused decode kernel only, whatever T: successive
 * launches of moe_layer_tokens_per_launch tokens (each reads the experts its
 * tokens chose).  Workspace as moe_layer_forward for T < 32. */
moe_status moe_layer_forward_chunked(const moe_config* cfg, const moe_layer_weights* wts,
                                     const void* x_bf16, const void* residual_bf16, int T,
                                     void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out,
                                     float* w_out, void* workspace, size_t ws_bytes,
                                     cudaStream_t stream);

/* The layer with the RMSNorm before it folded in, taking the residual
 * stream h_in itself (the normalisation that the per-layer GPU command
 * before the experts runs together with the router and the shared expert,
 * hakusoku "パイプライン概要"):
 *   x[t]      = bf16(h_in[t] / sqrt(mean(h_in[t]^2) + eps) * gamma_pre)
 *   then moe_layer_forward(x, residual = h_in).
 * gamma_pre bf16 [H] (device); h_in, x_out, h_out, y_norm bf16 [T][H], three
 * distinct buffers for h_in, x_out and h_out; x_out receives x.  The same eps
 * as the norm after the layer (cfg->eps).  The sum of squares is taken in
 * fp32.  For T < 32 tokens that one launch of the fused kernel takes (its
 * shared-memory plan then also holds gamma_pre; the count is that of
 * moe_layer_tokens_per_launch at hidden 4096) the norm runs inside that
 * kernel: its consumer warps normalise x in shared memory before the router
 * reads it.  Otherwise a norm kernel runs first, then moe_layer_forward.  Workspace,
 * errors and the remaining arguments as moe_layer_forward. */
moe_status moe_layer_forward_prenorm(const moe_config* cfg, const moe_layer_weights* wts,
                                     const void* gamma_pre_bf16, const void* h_in_bf16, int T,
                                     void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out,
                                     float* w_out, void* x_out_bf16, void* workspace, size_t ws_bytes,
                                     cudaStream_t stream);

/* Tokens one launch of the fused kernel takes for this shape on the current
 * device: the largest T <= min(8, 64 / K) whose shared-memory plan fits
 * (4 at hidden 4096, inter 1024, K = 4).  moe_layer_forward runs longer
 * batches in chunks of this size.  0 for an unsupported shape or when no
 * device is usable. */
int moe_layer_tokens_per_launch(const moe_config* cfg);

/* The same layer with the routing given instead of computed: idx int32
 * [T][K] (expert ids) and w fp32 [T][K] (their weights) in device memory,
 * typically the outputs of moe_router_topk.  The router weights
 * (wts->router_w, wts->router_bias) are not read and may be NULL; only
 * wts->expert_ptr[idx[t][k]] is read from the pointer table.  This is the
 * call of the expert-streaming tier, where the host must know the routing
 * first to bring the chosen experts into device memory (the pages' CPU reads
 * the GPU router's output, then reads the experts from SSD: "Flash-MoE:
 * ラップトップでの397Bパラメータモデルの実行", section "パイプライン概要").
 * An id outside [0, E) or a NULL / misaligned pointer for a chosen expert is
 * reported as MOE_ERR_DEVICE by moe_device_error.  Workspace: as
 * moe_layer_forward. */
moe_status moe_layer_forward_routed(const moe_config* cfg, const moe_layer_weights* wts,
                                    const void* x_bf16, const void* residual_bf16, int T,
                                    const int32_t* idx, const float* w, void* h_out_bf16,
                                    void* y_norm_bf16, void* workspace, size_t ws_bytes,
                                    cudaStream_t stream);

/* Allocation-free variant of moe_layer_forward.  The pages have no
 * counterpart: their engine owns all of its buffers.  It is for callers that
 * must not allocate device memory (a fixed memory budget, or a loop where
 * cudaMalloc -- which can synchronise the device and can fail under memory
 * pressure -- is not allowed) and that keep no workspace of their own: the
 * scratch is a MOE_NOALLOC_SCRATCH_BYTES area inside the library (a device
 * array of the loaded module), so the call allocates nothing.
 * Arguments and results are those of moe_layer_forward, without the
 * workspace.  A shape whose moe_layer_workspace_bytes exceeds
 * MOE_NOALLOC_SCRATCH_BYTES is rejected with MOE_ERR_WORKSPACE.
 * The first call on a device (with that device current) looks the scratch up
 * and zeroes its counters with synchronous CUDA calls: make it before any
 * stream capture.  All calls on a device share the one scratch, so calls that
 * may overlap in time (other streams, other host threads) race and must be
 * serialised by the caller.  Each call first clears the scratch's error word
 * on its stream (one 4-byte memset), so a device-side failure of one call (an
 * expired wait, a bad expert pointer) leaves only that call's outputs
 * unspecified; read it with moe_noalloc_device_error before the next call. */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
moe_status moe_layer_forward_noalloc(const moe_config* cfg, const moe_layer_weights* wts,
                                     const void* x_bf16, const void* residual_bf16, int T,
                                     void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out,
                                     float* w_out, cudaStream_t stream);

/* The device-side error of the last moe_layer_forward_noalloc call on the
 * current device: as moe_device_error (synchronises the stream, clears the
 * word), for the library's built-in scratch.  MOE_OK, MOE_ERR_TIMEOUT or
 * MOE_ERR_DEVICE; *detail (may be NULL) gets the raw code. */
moe_status moe_noalloc_device_error(uint32_t* detail, cudaStream_t stream);

/* Per-phase timing of one layer call, in the spirit of the pages' per-layer
 * --timing breakdown ("Flash-MoE: ...", section "パイプライン概要"): the same
 * computation as moe_layer_forward (idx/w outputs omitted), and every block
 * of the fused kernel writes global-timer stamps in ns to trace[block*128 + k]
 * (device memory, moe_layer_trace_blocks()*128 entries):
 * k = 0 start, 1 router rows done, 2 shared gate/up done, 3 routed gate/up
 * done, 4 shared wait done, 5 routed wait done, 6 last tile done, 7 arrived
 * on the final counter, 8 exit (for the last block to arrive: after it
 * normalised every row), 9 producer has the routing, 10 producer issued its last copy,
 * 11/12 first routed gate/up unit start/end, 13/14 first routed down unit
 * start/end; 16+2n / 17+2n: shared-memory tile n (n < 16) ready / released
 * by the consumers; 48+n: producer publishes tile n; sync warp: 64 x
 * prepared, 65 router barrier passed, 66 top-K done, 67 routing handed
 * over, 69 routed gate/up arrival, 71 routed barrier passed; 68 / 70 shared
 * gate/up arrival / barrier passed (written by the consumer warp that
 * handles that barrier).  Entries 80+k
 * (k < 8) hold poll counts (not times) of the block's waits: 0 consumers on
 * ring slots, 1 consumers on phase barriers, 2 consumers on x, 3 producer on
 * free slots, 4 producer on the routing, 5 sync warp on consumer arrivals,
 * 6 sync warp on grid barriers, 7 sync warp on x.  Unused entries are left
 * as they were.  Timestamps perturb nothing else. */
int moe_layer_trace_blocks(void);
moe_status moe_layer_forward_traced(const moe_config* cfg, const moe_layer_weights* wts,
                                    const void* x_bf16, const void* residual_bf16, int T,
                                    void* h_out_bf16, void* y_norm_bf16, void* workspace,
                                    size_t ws_bytes, uint64_t* trace, size_t trace_entries,
                                    cudaStream_t stream);

/* The same call with HOST activations: copies x and residual (host, pinned
 * for asynchronous copies) to device staging inside the workspace, runs the
 * layer, copies h_out and y_norm back to host, and synchronises the stream
 * before returning.  Workspace size: moe_layer_host_workspace_bytes. */
size_t moe_layer_host_workspace_bytes(const moe_config* cfg, int T);
moe_status moe_layer_forward_host(const moe_config* cfg, const moe_layer_weights* wts,
                                  const void* x_bf16_host, const void* residual_bf16_host,
                                  int T, void* h_out_bf16_host, void* y_norm_bf16_host,
                                  void* workspace, size_t ws_bytes, cudaStream_t stream);

/* The same without the final synchronisation: the copies and the layer are
 * enqueued on the stream and the call returns.  The host buffers must stay
 * valid and untouched, and the outputs are ready, only once the stream has
 * reached the end of the call (synchronise it, or wait on an event recorded
 * after it); on one stream, successive calls may share a workspace. */
moe_status moe_layer_forward_host_async(const moe_config* cfg, const moe_layer_weights* wts,
                                        const void* x_bf16_host, const void* residual_bf16_host,
                                        int T, void* h_out_bf16_host, void* y_norm_bf16_host,
                                        void* workspace, size_t ws_bytes, cudaStream_t stream);

/* The asynchronous host-buffer call with packed host buffers: xr_bf16_host
 * [2][T][H] holds x then residual, hy_bf16_host [2][T][H] receives h_out then
 * y_norm, so that each direction is one copy (when T*H*2 is a multiple of 256
 * bytes; two otherwise).  Same rules as moe_layer_forward_host_async. */
moe_status moe_layer_forward_host_packed(const moe_config* cfg, const moe_layer_weights* wts,
                                         const void* xr_bf16_host, int T, void* hy_bf16_host,
                                         void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Expert-streaming tier.  The pages keep all experts on SSD and read the 4
 * chosen ones per layer and token (toolarium, section "Mixture of Experts и
 * почему SSD достаточно"; hakusoku, section "パイプライン概要": parallel
 * pread of the K experts, about 2.4 ms of a 4.3 ms layer), leaning on the OS
 * page cache as the expert cache (toolarium, section "Flash-MoE: чистый C,
 * Metal и никакого Python"; hakusoku, section "試行錯誤と最適化": their own
 * cache measured slower than the page cache).  Here the store is pinned host
 * memory holding every expert of n_layers layers ([layer][expert] blobs of
 * moe_packed_expert_bytes each, contiguous), and the cache is n_slots
 * device slots of one blob each, keyed by (layer, expert) and replaced least
 * recently used.  Copies are cudaMemcpyAsync host -> device.
 *
 * Protocol per layer: moe_router_topk, read idx to the host,
 * moe_stream_resolve (brings in the misses, waits for pending prefetches,
 * fills the pointer table), then moe_layer_forward_routed on the same compute
 * stream with that table.  moe_stream_prefetch, on another stream, may bring
 * in the experts predicted for a later layer meanwhile (the streaming
 * implementations that the blog.cecily.jp article on BigMoeOnEdge describes
 * rely on knowing the next layer's experts before the current layer ends;
 * the pages' Mac engine measured its prefetch and speculative variants as
 * losses there: hakusoku, section "試行錯誤と最適化").  The slots that a
 * resolve call hands out stay resident until
 * the next resolve call on the cache, which records on its compute stream
 * that they may be reused: enqueue the layer that reads them on that stream
 * before the next resolve.  A cache is used by one host thread at a time
 * (calls lock it). */
typedef struct moe_stream_cache moe_stream_cache;

/* Creates a cache: allocates n_slots * moe_packed_expert_bytes of device
 * memory (the one call of the library that allocates device memory) and two
 * CUDA events per slot.  host_pinned_experts (store_bytes long) must hold
 * n_layers * n_experts blobs in page-locked memory (cudaHostAlloc /
 * cudaHostRegister) and stay valid until destroy.  MOE_ERR_OOM if the slots
 * do not fit; MOE_ERR_INVALID_ARG for a store shorter than the blobs need or
 * not page-locked (both ends are checked), n_layers < 1 or n_slots < 1. */
moe_status moe_stream_create(const moe_config* cfg, int n_layers, const void* host_pinned_experts,
                             size_t store_bytes, int n_slots, moe_stream_cache** out);

/* A cache whose store is a file instead of pinned memory: the file at `path`
 * holds the same n_layers * n_experts blobs ([layer][expert], each
 * moe_packed_expert_bytes long) -- the pages' own tier: experts on SSD, the
 * K chosen ones read with parallel pread per layer ("Flash-MoE: чистый C,
 * Metal и никакого Python", toolarium.ru; hakusoku.com, section
 * "パイプライン概要").  Every fill of a prefetch or resolve call is read with
 * pread on a pool of n_read_threads host threads, in parallel, into one of 16
 * pinned staging buffers, then copied to its slot on the call's stream; the
 * call returns once its reads are done (the copies are asynchronous).
 * direct_io = 1 opens the file with O_DIRECT (bypassing the OS page cache;
 * needs blobs of a multiple of 4096 bytes), 0 reads through the page cache.
 * A staging buffer is reused once its copy has completed (the host waits
 * for that).  MOE_ERR_IO if the file cannot be opened or a read fails (the
 * slot is left empty); MOE_ERR_INVALID_ARG for a file shorter than the blobs
 * need.  Everything else as moe_stream_create. */
moe_status moe_stream_create_file(const moe_config* cfg, int n_layers, const char* path, int direct_io,
                                  int n_slots, int n_read_threads, moe_stream_cache** out);

/* Reads done by a file-backed cache since create: count, bytes and the host
 * time the calls spent in them (parallel reads of one call count once). */
moe_status moe_stream_file_stats(const moe_stream_cache* cache, uint64_t* reads, uint64_t* read_bytes,
                                 double* read_ms);

/* Enqueues on copy_stream the copies of those of expert_ids_host[0..n)
 * (experts of `layer`) that are not resident, each into the least recently
 * used slot that no resolve call holds; the copy waits for the last kernel
 * that read the slot.  A hint: ids that find no free slot are skipped
 * (counted in prefetch_dropped).  Does not synchronise.  MOE_ERR_IO if a
 * copy cannot be enqueued (its slot is left empty; the ids after it are not
 * looked at). */
moe_status moe_stream_prefetch(moe_stream_cache* cache, int layer, const int32_t* expert_ids_host,
                               int n, cudaStream_t copy_stream);

/* Makes the distinct experts of idx_host[0..n) (experts of `layer`)
 * resident: misses are copied on compute_stream, and compute_stream waits
 * for prefetch copies still in flight.  Then writes expert_ptr_dev (device
 * array [E] of device pointers) on compute_stream: the slot of every
 * resolved expert; other entries are unspecified.  MOE_ERR_OOM if the
 * distinct ids outnumber the slots; MOE_ERR_IO if a miss cannot be copied
 * (the table is not written, the slots of this call are released, the cache
 * stays usable).  Does not synchronise the device, but blocks the calling
 * thread when 8 resolves are still in flight (its pinned staging ring), so it
 * must not be called while compute_stream is being captured. */
moe_status moe_stream_resolve(moe_stream_cache* cache, int layer, const int32_t* idx_host, int n,
                              const void** expert_ptr_dev, cudaStream_t compute_stream);

/* The same resolve decided on the GPU, for routing that stays on the device:
 * idx_dev (device int32 [n], n <= 64, typically moe_router_topk's output)
 * names experts of `layer`.  One kernel looks each distinct id up in a
 * device-resident slot table (hits touch nothing else), picks for every
 * miss the slot the host policy would pick (an empty slot, lowest index
 * first, else the least recently used one not taken by this call), updates
 * the table, and writes expert_ptr_dev[e] for every id; a second kernel
 * copies the missed experts from the pinned host store into their slots
 * with 16-byte loads of mapped host memory (it returns at once when nothing
 * missed).  Nothing waits on the host and nothing is read back, so a layer's
 * router, this call and moe_layer_forward_routed can run back to back or be
 * captured into a CUDA graph; the pages' CPU reads the router output before
 * its reads (hakusoku "パイプライン概要"), which this call keeps on the GPU.
 * A cache serves either this call or moe_stream_resolve/moe_stream_prefetch,
 * whichever is called first (the other then returns MOE_ERR_INVALID_ARG);
 * MOE_ERR_UNSUPPORTED for a file store or a host store the device cannot map.
 * Ids outside [0, E) get no table entry (the layer then reports a bad
 * pointer); more distinct ids than slots leave MOE_ERR_OOM in the cache's
 * device error word (moe_stream_stats' device_error) and the table
 * unwritten.  moe_stream_stats and moe_stream_copy_timing read the device
 * counters back (synchronising); bytes_h2d counts the bytes the fill kernel
 * copied and the copy timing reports its busy time from device timestamps. */
moe_status moe_stream_resolve_device(moe_stream_cache* cache, int layer, const int32_t* idx_dev, int n,
                                     const void** expert_ptr_dev, cudaStream_t stream);

/* One streamed layer in one launch: moe_layer_forward (router, top-K, the
 * chosen experts' SwiGLU FFNs, shared expert, combine, residual, RMSNorm;
 * same arguments, outputs and workspace) with the routed experts taken from
 * `cache` (layer `layer`) instead of wts->expert_ptr, which is ignored.
 * Inside the launch, the block that finds the routing applies the device
 * resolve's policy to the T*K chosen experts (hits touch their slots; a miss
 * takes the lowest empty slot not held by this call, else the least
 * recently used one, and is mapped to it), then every block copies its
 * share of the missed blobs from the pinned host store (mapped host memory,
 * 16-byte loads) into their slots and waits for the others before the
 * routed weights are read.  So the stand-alone router, the resolve and the
 * fill launches of moe_stream_resolve_device are not needed, and the
 * routing never leaves the GPU (hakusoku "パイプライン概要" reads the GPU's
 * routing on the CPU before its expert reads; blog.cecily.jp on BigMoeOnEdge
 * streams the routed experts of each layer on demand).  The cache follows
 * the same rules as moe_stream_resolve_device (this call and that one may
 * share a cache); it must have at most 32767 slots and at most 64 per
 * expert of a layer, and E <= 65535 (MOE_ERR_UNSUPPORTED otherwise), and
 * must live on the current device with blobs of this layer's shape
 * (MOE_ERR_INVALID_ARG).  Counters: as moe_stream_resolve_device (hits,
 * misses, bytes_h2d; no copy timing).  More distinct experts in one launch
 * than slots: MOE_ERR_OOM in the cache's device error word, the call's
 * assignments undone, and the layer's device error word (moe_device_error)
 * reports a bad expert pointer; its outputs are then not written.  Tokens
 * beyond one launch's limit (64 / K) run in successive launches, each
 * resolving its own experts.  A launch changes the cache's tables and slots:
 * calls that share a cache (this one, moe_stream_resolve_device and the
 * layers reading its slots) must be ordered, e.g. on one stream. */
moe_status moe_layer_forward_streamed(const moe_config* cfg, const moe_layer_weights* wts, const void* x_bf16,
                                      const void* residual_bf16, int T, void* h_out_bf16, void* y_norm_bf16,
                                      int32_t* idx_out, float* w_out, moe_stream_cache* cache, int layer,
                                      void* workspace, size_t ws_bytes, cudaStream_t stream);

/* Counters since create: resolved experts found resident (hits) or copied
 * on demand (misses), prefetch copies issued, resolved experts that a
 * prefetch had brought in and no resolve had used yet (prefetch_hits),
 * prefetch ids skipped for want of a free slot, and bytes copied. */
typedef struct {
  uint64_t hits, misses, prefetches, prefetch_hits, prefetch_dropped, bytes_h2d;
  uint64_t device_error;  /* device-resolved caches: 0, or the first error a resolve kernel met */
} moe_stream_counters;
moe_status moe_stream_stats(const moe_stream_cache* cache, moe_stream_counters* out);

/* Waits for the cache's copies and kernels that may still use its slots
 * (synchronises the device), then frees the slots and events. */
void moe_stream_destroy(moe_stream_cache* cache);

/* Timing of the host-to-device copies (a measurement aid; none on the
 * pages): once enabled, every copy the cache issues is bracketed by a pair of
 * CUDA events on its stream.  moe_stream_copy_timing waits for the timed
 * copies, returns the time the link was busy with them (the union of their
 * intervals; copies on the prefetch and compute streams may overlap), the
 * sum of their durations, their count and bytes, and starts over. */
typedef struct {
  double busy_ms, copy_ms;
  uint64_t copies, bytes;
} moe_stream_copy_times;
moe_status moe_stream_enable_copy_timing(moe_stream_cache* cache, int on);
moe_status moe_stream_copy_timing(moe_stream_cache* cache, moe_stream_copy_times* out);

/* Host-side fault injection for tests of the streaming tier's error paths
 * (no counterpart on the pages; nothing is done to the GPU):
 *   MOE_FAULT_COPY:  the copy issued after `countdown` more copies on this
 *                    cache reports failure instead of being enqueued (the
 *                    calling prefetch or resolve returns MOE_ERR_IO);
 *   MOE_FAULT_ALLOC: the next moe_stream_create's slot allocation reports
 *                    failure (MOE_ERR_OOM); cache may be NULL;
 *   MOE_FAULT_NONE:  clears both. */
enum { MOE_FAULT_NONE = 0, MOE_FAULT_COPY = 1, MOE_FAULT_ALLOC = 2 };
moe_status moe_stream_inject_fault(moe_stream_cache* cache, int what, int countdown);

/* Read (synchronising the stream) and clear the device-side error word of a
 * layer workspace.  Returns MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE;
 * *detail (may be NULL) gets the raw code. */
moe_status moe_device_error(void* workspace, uint32_t* detail, cudaStream_t stream);

/* Self-test of the bounded device-side wait (no counterpart on the pages):
 * launches a tiny kernel that waits, with the given limit in nanoseconds, on
 * a counter of the workspace that nothing increments.  The wait must give up,
 * record MOE_ERR_TIMEOUT in the workspace's error word (read it with
 * moe_device_error) and return, leaving the GPU context usable.  The first
 * 256 bytes of the workspace must be zero (moe_workspace_init). */
moe_status moe_selftest_bounded_wait(void* workspace, size_t ws_bytes, uint64_t timeout_ns,
                                     cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif
