/*
 * zimage_dit.h -- C ABI of the B200 (sm_100a) Z-Image S3-DiT forward library.
 *
 * What it computes (page title, section):
 *   - ostris ai-toolkit docs "Z-Image", sections "Architecture" and "Latent
 *     space": a single-stream DiT; text and 2x2-patchified image tokens share
 *     one sequence; 2 noise-refiner blocks (image tokens), 2 context-refiner
 *     blocks (text tokens, unmodulated) and 30 main blocks; hidden 3840 =
 *     30 heads x 128; SwiGLU FFN 10240; RMSNorm and QK-RMSNorm; 3-axis RoPE
 *     [32, 48, 48] with theta 256; adaLN modulation from a 256-d timestep
 *     embedding.
 *   - z-image-turbo-mnn model card, "Conversion details": the attention output
 *     projection and FFN w2 feed an RMSNorm directly (post-norms); "Model
 *     files": transformer(sample [1,16,H/8,W/8], timestep [1], text features
 *     [1,L,2560]) -> output of the sample's shape; "Scheduler": FlowMatch
 *     Euler with shift 3.0, sigmas linspace(1, 1/N, N) shifted, timestep
 *     passed as 1 - sigma, model output negated before the Euler step.
 *   - FastVideo zimage handoff, "Pinned official pipeline context": a
 *     num_steps + 1 schedule ending at sigma 0, the final zero-sigma call skipped.
 * Readings of points the pages leave open are fixed in the library and listed
 * in the design notes; the same readings define the CPU oracle in the tests.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless the argument name starts
 *     with h_.  The caller owns every buffer and the stream; the library never
 *     allocates or frees device memory and never synchronises the stream.
 *     Pointers must stay valid until the enqueued work has completed.
 *   - bf16 tensors are passed as uint16_t bit patterns.  Weights are row-major
 *     in the checkpoint's [out, in] orientation.
 *   - Device pointers to bf16 matrices and to fp32 activations must be 16-byte
 *     aligned (TMA and vector loads); otherwise ZI_ERR_ALIGN.
 *   - Every call validates its arguments before enqueuing anything and returns
 *     a status (0 = ZI_OK, negative = error); nothing is enqueued on error.
 *     Asynchronous device failures (a pipeline wait that ran out) are reported
 *     later by zi_device_status().
 *   - There is no CPU fallback: calls that launch kernels fail with
 *     ZI_ERR_DEVICE unless the current device is compute capability 10.0.
 */
#ifndef ZIMAGE_DIT_H
#define ZIMAGE_DIT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZI_API __attribute__((visibility("default")))
#else
#define ZI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st* zi_stream_t;

enum zi_status {
  ZI_OK = 0,
  ZI_ERR_ARG = -1,       /* null pointer, bad enum, negative size */
  ZI_ERR_SHAPE = -2,     /* sizes the kernels do not support */
  ZI_ERR_ALIGN = -3,     /* pointer or stride not 16-byte aligned */
  ZI_ERR_WORKSPACE = -4, /* workspace missing or smaller than zi_*_workspace_size() */
  ZI_ERR_CUDA = -5,      /* a CUDA runtime/driver call failed (launch error etc.) */
  ZI_ERR_TIMEOUT = -6,   /* a kernel's bounded pipeline wait ran out (zi_device_status) */
  ZI_ERR_DEVICE = -7,    /* current device is not an sm_100 GPU */
  ZI_ERR_SCRATCH_LIMIT = -8 /* sizes need more than ZI_STATIC_SCRATCH_BYTES (zi_block_forward_noalloc) */
};

/* Sizes of one model variant.  zi_config_default() gives Z-Image's
 * (ostris "Z-Image", "Architecture"; numbers checked against the 6.15B /
 * 521-key totals of "Components" and the FastVideo "Transformer" notes). */
typedef struct zi_config {
  int dim;          /* D, hidden width (3840); multiple of 256 */
  int heads;        /* attention heads (30); dim == heads * head_dim */
  int head_dim;     /* 128 (the only supported value) */
  int ffn;          /* SwiGLU inner width F (10240) */
  int cap_dim;      /* text-feature width (2560) */
  int t_freq;       /* sinusoidal timestep width (256, the only supported value) */
  int t_mid;        /* timestep MLP hidden width (1024; multiple of 8) */
  int in_ch;        /* latent channels (16) */
  int patch;        /* 2 (the only supported value) */
  int n_noise;      /* noise-refiner blocks (2) */
  int n_ctx;        /* context-refiner blocks (2) */
  int n_main;       /* main blocks (30) */
  int rope_axes[3]; /* {32, 48, 48}; sum == head_dim, each even */
  float rope_theta; /* 256 */
  float norm_eps;   /* every RMSNorm (1e-5) */
  float final_eps;  /* final LayerNorm (1e-6) */
  float t_scale;    /* model timestep t in [0,1] is scaled by this (1000) before the sinusoid */
} zi_config;

/* Weights of one block (device pointers, bf16).  D = dim, F = ffn,
 * Fp = ffn rounded up to a multiple of 128 (zi_ffn_padded). */
typedef struct zi_block_weights {
  const uint16_t* w_qkv;   /* [3D, D]: rows of to_q, then to_k, then to_v (zi_pack_qkv) */
  const uint16_t* w_out;   /* [D, D]  attention output projection */
  const uint16_t* w13;     /* [2Fp, D]: w1 and w3 interleaved in 128-row groups (zi_pack_ffn) */
  const uint16_t* w2;      /* [D, Fp]: w2 with zero columns F..Fp (zi_pack_ffn) */
  const uint16_t* g_attn1; /* [D] pre-attention RMSNorm gain */
  const uint16_t* g_attn2; /* [D] post-attention RMSNorm gain */
  const uint16_t* g_ffn1;  /* [D] pre-FFN RMSNorm gain */
  const uint16_t* g_ffn2;  /* [D] post-FFN RMSNorm gain */
  const uint16_t* g_q;     /* [head_dim] QK-RMSNorm gains, shared by all heads */
  const uint16_t* g_k;     /* [head_dim] */
  const uint16_t* w_ada;   /* [4D, min(D,256)] adaLN linear, or NULL for an unmodulated block */
  const uint16_t* b_ada;   /* [4D] its bias (NULL iff w_ada is NULL) */
  /* Optional e4m3 projections (all four, or all NULL).  When set, the block's QKV
   * and FFN w1|w3 projections run on the tensor cores in e4m3 (kind::f8f6f4)
   * from these instead of w_qkv / w13, and the norms feeding them emit e4m3
   * activations with one scale per token row (zi_quantize_rows_e4m3 gives the
   * recipe; its header comment states it).  The pages' quantised builds (ostris
   * "Z-Image", "Specifics"; H3ddle "What was changed, and why") are the prior art. */
  const uint8_t* w_qkv8;   /* [3D, D] e4m3 codes of w_qkv, one scale per row ... */
  const float* s_qkv;      /* [3D] ... these (zi_quantize_rows_e4m3 of w_qkv) */
  const uint8_t* w13_8;    /* [2Fp, D] e4m3 codes of w13 */
  const float* s_13;       /* [2Fp] */
  /* Optional, with the four above (all four, or all NULL): the output projection
   * and FFN w2 in e4m3 too.  The attention output and the SwiGLU output are then
   * quantised per row (the same recipe) by an extra pass before each GEMM. */
  const uint8_t* w_out8;   /* [D, D] e4m3 codes of w_out */
  const float* s_out;      /* [D] */
  const uint8_t* w2_8;     /* [D, Fp] e4m3 codes of w2 (zero columns F..Fp) */
  const float* s_2;        /* [D] */
} zi_block_weights;

/* Weights of the whole transformer.  The block arrays are HOST arrays (of
 * structs holding device pointers) of n_noise / n_ctx / n_main entries. */
typedef struct zi_model_weights {
  const uint16_t* x_emb_w;   /* [D, 4*in_ch]  x_embedder */
  const uint16_t* x_emb_b;   /* [D] */
  const uint16_t* cap_norm;  /* [cap_dim]  cap_embedder RMSNorm gain */
  const uint16_t* cap_w;     /* [D, cap_dim] */
  const uint16_t* cap_b;     /* [D] */
  const uint16_t* t_w1;      /* [t_mid, t_freq] */
  const uint16_t* t_b1;      /* [t_mid] */
  const uint16_t* t_w2;      /* [min(D,256), t_mid] */
  const uint16_t* t_b2;      /* [min(D,256)] */
  const uint16_t* final_ada_w; /* [D, min(D,256)] final layer adaLN (applied to SiLU(c)) */
  const uint16_t* final_ada_b; /* [D] */
  const uint16_t* final_w;   /* [4*in_ch, D] final_layer.linear */
  const uint16_t* final_b;   /* [4*in_ch] */
  const zi_block_weights* noise; /* host array [n_noise], modulated */
  const zi_block_weights* ctx;   /* host array [n_ctx], w_ada == NULL */
  const zi_block_weights* main;  /* host array [n_main], modulated */
  const uint16_t* cap_pad;   /* [D] cap_pad_token: embedding of padded text rows
                                (read by zi_model_forward_varlen only; may be NULL otherwise) */
} zi_model_weights;

/* Human-readable text of a status code (static storage). */
ZI_API const char* zi_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
ZI_API int zi_version(void);

/* Fill *cfg with Z-Image's sizes (see zi_config).  ZI_ERR_ARG if cfg is NULL. */
ZI_API int zi_config_default(zi_config* cfg);

/* ffn rounded up to a multiple of 128 (the interleave group of w13). */
ZI_API int zi_ffn_padded(int ffn);

/* ---------------------------------------------------------------- weight layout
 * Library-owned layout steps, enqueued on `stream` as device copies. */

/* w_qkv[0:D] = wq, [D:2D] = wk, [2D:3D] = wv; each [D, D]. */
ZI_API int zi_pack_qkv(const uint16_t* wq, const uint16_t* wk, const uint16_t* wv, int dim, uint16_t* w_qkv,
                zi_stream_t stream);

/* w13 [2Fp, D]: group g (128 rows) of w1 goes to rows [256g, 256g+128) and
 * group g of w3 to rows [256g+128, 256g+256); rows past F in a group are zero.
 * w2p [D, Fp] = w2 [D, F] with zero columns F..Fp.  Lets one 256-wide GEMM
 * tile hold matching gate and up columns for the fused SwiGLU. */
ZI_API int zi_pack_ffn(const uint16_t* w1, const uint16_t* w3, const uint16_t* w2, int ffn, int dim, uint16_t* w13,
                uint16_t* w2p, zi_stream_t stream);

/* ---------------------------------------------------------------- workspaces */

/* Bytes of workspace zi_block_forward needs for batch x seq tokens. */
ZI_API int zi_block_workspace_size(const zi_config* cfg, int batch, int seq, size_t* h_bytes);

/* Bytes of workspace zi_model_forward (and zi_model_forward_varlen) needs for
 * batch x (s_img + s_txt) tokens, s_img = (lat_h/2)(lat_w/2). */
ZI_API int zi_model_workspace_size(const zi_config* cfg, int batch, int lat_h, int lat_w, int s_txt, size_t* h_bytes);

/* ---------------------------------------------------------------- the forward */

/* One S3-DiT block (ostris "Z-Image", "Architecture"; post-norms per the
 * z-image-turbo-mnn card, "Conversion details") on x [batch, seq, D] fp32:
 *   h = RMSNorm1(x)(1 + scale_msa); q, k, v = h Wqkv; q, k <- RoPE(QKRMSNorm(.));
 *   x += tanh(gate_msa) RMSNorm2(Attn(q, k, v) Wout);
 *   h = RMSNormF1(x)(1 + scale_mlp); x += tanh(gate_mlp) RMSNormF2(W2(SiLU(W1 h) * W3 h)),
 * with [scale_msa, gate_msa, scale_mlp, gate_mlp] = w_ada c + b_ada.
 * Unmodulated blocks (w->w_ada == NULL) use scale 0 and gate 1; d_c may then be NULL.
 *   d_c    fp32 [batch, min(D,256)] conditioning vector (t-embedder output)
 *   d_pos  int32 [seq, 3] position ids of one sequence (shared by the batch)
 *   d_x_in / d_x_out  fp32 [batch, seq, D]; may be the same buffer
 *   d_ws   workspace of at least zi_block_workspace_size() bytes (256-byte aligned)
 * Attention is non-causal over the seq tokens of each batch element. */
ZI_API int zi_block_forward(const zi_config* cfg, const zi_block_weights* w, const float* d_c, const int32_t* d_pos,
                     int batch, int seq, const float* d_x_in, float* d_x_out, void* d_ws, size_t ws_bytes,
                     zi_stream_t stream);

/* Full transformer forward (z-image-turbo-mnn "Model files" interface):
 *   d_latent fp32 [batch, in_ch, lat_h, lat_w] (lat_h, lat_w even)
 *   d_t      fp32 [batch] model timestep, 1 = clean (pass 1 - sigma')
 *   d_txt    bf16 [batch, s_txt, cap_dim] text features
 *   d_out    fp32 [batch, in_ch, lat_h, lat_w] raw model output (not negated)
 * Sequence per batch element: [(lat_h/2)(lat_w/2) image tokens; s_txt text tokens],
 * image tokens refined by the noise refiners, text tokens by the context
 * refiners, then all tokens through the main blocks and image tokens through
 * the final layer.  s_txt >= 1; every text row is a real token (no padding;
 * for a batch of prompts of different lengths use zi_model_forward_varlen). */
ZI_API int zi_model_forward(const zi_config* cfg, const zi_model_weights* w, int batch, int lat_h, int lat_w, int s_txt,
                     const float* d_latent, const float* d_t, const uint16_t* d_txt, float* d_out, void* d_ws,
                     size_t ws_bytes, zi_stream_t stream);

/* zi_model_forward for a batch whose prompts differ in length (FastVideo zimage
 * handoff, "Transformer": a padded variable-length stream needs a key mask;
 * ostris "Z-Image", "Architecture": the checkpoint's cap_pad_token).  Element b
 * holds h_txt_len[b] real text tokens followed by s_txt - h_txt_len[b] padding
 * rows of d_txt (their contents are ignored):
 *   - padding rows take w->cap_pad as their embedding (after the cap embedder);
 *   - padding rows are removed from the keys of every attention (context
 *     refiners and main blocks), i.e. an additive -inf key mask; the image rows
 *     and real text rows then see exactly their unpadded sequence;
 *   - positions follow each element's own length: image token (r, c) ->
 *     (h_txt_len[b] + 1, r, c), text row j -> (j + 1, 0, 0) (a reading; it makes
 *     the output for element b equal to a batch-1 forward on its unpadded text).
 *   h_txt_len  HOST int32 [batch], each in [1, s_txt]; otherwise ZI_ERR_ARG.
 * Other arguments as for zi_model_forward; w->cap_pad must be non-NULL.  The
 * lengths reach the device as kernel arguments (no host-to-device copy), so the
 * call can be captured in a CUDA graph. */
ZI_API int zi_model_forward_varlen(const zi_config* cfg, const zi_model_weights* w, int batch, int lat_h, int lat_w,
                                   int s_txt, const int32_t* h_txt_len, const float* d_latent, const float* d_t,
                                   const uint16_t* d_txt, float* d_out, void* d_ws, size_t ws_bytes,
                                   zi_stream_t stream);

/* zi_model_forward that also copies the residual stream after every block into
 * d_trace, fp32 [n_noise + n_ctx + n_main][rows][dim] in the library's row order
 * (rows = batch * s_img image rows, then batch * s_txt text rows; blocks in
 * execution order: noise refiners, context refiners, main blocks).  The kernels
 * and their launch shapes are those of zi_model_forward; the copies are extra.
 * Used to check every block of a full-size forward against a reference. */
ZI_API int zi_model_forward_trace(const zi_config* cfg, const zi_model_weights* w, int batch, int lat_h, int lat_w,
                                  int s_txt, const float* d_latent, const float* d_t, const uint16_t* d_txt,
                                  float* d_out, float* d_trace, void* d_ws, size_t ws_bytes, zi_stream_t stream);

/* FlowMatch-Euler step in place (z-image-turbo-mnn "Scheduler"):
 *   y = d_out_uncond ? d_out_uncond + guidance (d_out_cond - d_out_uncond) : d_out_cond
 *   d_x += (sigma_next - sigma) * (-y)          (n fp32 elements)
 * d_out_uncond may be NULL (no CFG; guidance ignored).  n == 0 enqueues nothing and
 * returns ZI_OK whatever the pointers; n above 256 (2^31 - 1) returns ZI_ERR_SHAPE. */
ZI_API int zi_euler_step(float* d_x, const float* d_out_cond, const float* d_out_uncond, float guidance, double sigma,
                  double sigma_next, size_t n, zi_stream_t stream);

/* Host helper: the n_steps + 1 shifted sigmas, sigma'_i = shift s / (1 + (shift-1) s)
 * for s = linspace(1, 1/n_steps, n_steps), then 0 (z-image-turbo-mnn "Scheduler";
 * FastVideo handoff "Scheduler").  h_sigmas has n_steps + 1 entries. */
ZI_API int zi_sigmas(int n_steps, double shift, double* h_sigmas);

/* Host helper: the model timestep of each of the n_steps transformer calls of that
 * schedule, t_i = 1 - sigma'_i (1 = clean), formed in double and rounded to float
 * once: the card passes (1000 - 1000 sigma') / 1000 to the transformer
 * (z-image-turbo-mnn "Scheduler"), and the zero-sigma end point gets no call
 * (FastVideo handoff "Pinned official pipeline context").  h_t has n_steps
 * entries, ready to copy into zi_model_forward's d_t.  ZI_ERR_ARG if n_steps <= 0,
 * shift <= 0 or h_t is NULL. */
ZI_API int zi_timesteps(int n_steps, double shift, float* h_t);

/* ---------------------------------------------------------------- fixed-scratch variant
 * The pages describing the method have no counterpart to this entry point; it
 * exists for callers that cannot allocate device memory.  Examples: a plugin
 * running inside a host program whose memory manager owns all device memory
 * and hands plugins no allocator, or a latency-critical loop that forbids
 * cudaMalloc after start-up (cudaMalloc can synchronise the device and stall
 * other work).  Such callers cannot provide the workspace zi_block_forward needs. */

/* Bytes of the library's fixed device scratch (128 MiB).  Every GPU that loads the
 * library holds this much device memory until the process exits. */
#define ZI_STATIC_SCRATCH_BYTES (128u * 1024u * 1024u)

/* zi_block_forward without a workspace argument: the scratch is a file-scope
 * device array of ZI_STATIC_SCRATCH_BYTES inside the library.  The caller still
 * passes (and owns) the inputs and the output; arguments mean what they mean
 * for zi_block_forward.
 *   - Allocates nothing: no cudaMalloc/cudaFree and no allocating library call.
 *   - Sizes whose zi_block_workspace_size() exceeds ZI_STATIC_SCRATCH_BYTES are
 *     rejected with ZI_ERR_SCRATCH_LIMIT before anything is enqueued (about 1,350
 *     tokens of batch x seq at Z-Image's full width).
 *   - The first call on each device looks up the scratch's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it for later
 *     calls; make that first call before any stream capture on that device.
 *     cudaDeviceReset destroys the array with the context, so the kept address
 *     is stale afterwards: do not call this entry point on a device that was
 *     reset earlier in the same process.
 *   - Every call on a device shares the one scratch array, and it keeps the last
 *     call's contents.  Nothing in it needs to start at zero (each call writes
 *     every scratch byte it reads), but calls whose GPU work overlaps -- on
 *     different streams, or from different host threads -- race on the scratch
 *     and corrupt each other's results: serialise them. */
ZI_API int zi_block_forward_noalloc(const zi_config* cfg, const zi_block_weights* w, const float* d_c,
                                    const int32_t* d_pos, int batch, int seq, const float* d_x_in, float* d_x_out,
                                    zi_stream_t stream);

/* ---------------------------------------------------------------- single steps
 * The steps zi_block_forward / zi_model_forward chain, exposed for testing and
 * for callers that schedule the pieces themselves. */

/* Position ids of one sequence [image; text] (3-axis RoPE, ostris "Architecture";
 * the id scheme is a reading): image token (r, c) of a grid_h x grid_w grid
 * -> (s_txt + 1, r, c); text token j -> (j + 1, 0, 0).  d_pos int32 [grid_h*grid_w + s_txt, 3]. */
ZI_API int zi_positions(int s_txt, int grid_h, int grid_w, int32_t* d_pos, zi_stream_t stream);

/* RoPE table for n tokens: d_cos_sin fp32 [n, head_dim/2, 2] holding (cos, sin) of
 * pos[axis] * theta^(-2j/d_axis) for rotation pair j (pairs of axis 0 first). */
ZI_API int zi_rope_table(const zi_config* cfg, const int32_t* d_pos, int n, float* d_cos_sin, zi_stream_t stream);

/* C[M, N] = A[M, K] B[N, K]^T, bf16 in, fp32 accumulate, bf16 out (tcgen05).
 * K % 64 == 0, N % 256 == 0, M >= 1; rows are contiguous (strides K and N).
 * Same kernel as the projections of the forward (128 x 256 tiles on persistent
 * CTAs).  Inside the forward the ragged last wave of tiles is cut along K into
 * pieces whose fp32 partials the last-arriving piece sums in piece order; this
 * entry point has no workspace for those partials, so its tiles always run whole. */
ZI_API int zi_gemm_bf16(const uint16_t* d_a, const uint16_t* d_b, uint16_t* d_c, int m, int n, int k,
                        zi_stream_t stream);

/* zi_gemm_bf16 on CTA pairs: two CTAs of a cluster on two SMs compute each 256 x 256
 * output tile with one tcgen05 cta_group::2 instruction stream (A rows split between
 * them, B split along N), so each SM stages 32 KB of operands per 64-deep k-block
 * instead of 48 KB.  Same arguments, restrictions and result as zi_gemm_bf16; the
 * forward picks per projection whichever of the two kernels suits its shape. */
ZI_API int zi_gemm_bf16_pair(const uint16_t* d_a, const uint16_t* d_b, uint16_t* d_c, int m, int n, int k,
                             zi_stream_t stream);

/* Per-row e4m3 quantisation (OCP e4m3: bias 7, 3 mantissa bits, max 448):
 *   s[r] = amax_r / 448 (fp32), q[r][k] = e4m3(x[r][k] * (448 / amax_r)), the
 *   product formed in fp32, rounded to nearest even, saturating at +-448; a row of
 *   zeros gets s = 1 and zero codes.  The same recipe the norms use for e4m3 blocks.
 *   d_x   [rows, cols] fp32 (x_bf16 = 0) or bf16 (x_bf16 = 1), contiguous
 *   d_q   [rows, cols] uint8 codes;  d_s [rows] fp32 scales
 * cols % 4 == 0 and cols <= 16384 (ZI_ERR_SHAPE otherwise); 16-byte aligned pointers.
 * Weights for e4m3 blocks are made with it (rows = output channels). */
ZI_API int zi_quantize_rows_e4m3(const void* d_x, int x_bf16, int rows, int cols, uint8_t* d_q, float* d_s,
                                 zi_stream_t stream);

/* C[M, N] = bf16( sa[m] sb[n] sum_k A[m, k] B[n, k] ), A and B e4m3 codes (row-major,
 * K contiguous), sa [M] / sb [N] their per-row scales; fp32 accumulation on
 * tcgen05 (kind::f8f6f4).  K % 128 == 0, N % 256 == 0. */
ZI_API int zi_gemm_e4m3(const uint8_t* d_a, const float* d_sa, const uint8_t* d_b, const float* d_sb, uint16_t* d_c,
                        int m, int n, int k, zi_stream_t stream);

/* Non-causal softmax(q k^T / sqrt(128)) v per head over seq tokens per batch element.
 * d_qkv bf16 [batch*seq, 3*heads*128] (q | k | v, head h at columns h*128 of each);
 * d_out bf16 [batch*seq, heads*128]. */
ZI_API int zi_attention(const uint16_t* d_qkv, uint16_t* d_out, int batch, int seq, int heads, zi_stream_t stream);

/* zi_attention with a key mask: element b attends to its first d_kv_len[b] keys
 * only (rows past them are padding; FastVideo zimage handoff, "Transformer").
 * Every query row is still computed.  d_kv_len DEVICE int32 [batch]; values
 * are clamped to [1, seq] on the device. */
ZI_API int zi_attention_varlen(const uint16_t* d_qkv, uint16_t* d_out, int batch, int seq, int heads,
                               const int32_t* d_kv_len, zi_stream_t stream);

/* Test hook for the attention softmax's second exponential: d_y[i] = 2^d_x[i] as the
 * attention kernel computes it on the FMA pipe for 3 of every 8 score pairs (the rest
 * go to the MUFU ex2 unit), so that its accuracy can be checked directly.  The method
 * (the FMA-pipe exponential of FlashAttention-4, restated): x is clamped at -126;
 * Cody-Waite split x = n + f with n = rint(x) (by adding and subtracting 1.5 * 2^23)
 * and f in [-1/2, 1/2]; 2^f from a degree-3 polynomial whose coefficients are a
 * minimax fit of the relative error on [-1/2, 1/2] (Remez exchange); n is added to
 * the result's exponent field.  Maximum relative error 7.5e-5 for x in [-125, 0],
 * below the bf16 rounding the probabilities get next; below -125 (where the result
 * can fall into the denormal range; a masked key's -inf included) it gives a value
 * in [0, 2^-124].  d_x, d_y fp32 [n]; n == 0 enqueues nothing; n above 512 (2^31 - 1)
 * returns ZI_ERR_SHAPE. */
ZI_API int zi_exp2_poly(const float* d_x, float* d_y, size_t n, zi_stream_t stream);

/* ---------------------------------------------------------------- launch profiling */

/* Kernel identities reported by zi_profile_end. */
enum zi_kernel_kind {
  ZI_KERNEL_GEMM_QKV = 1,       /* QKV projection + QK-RMSNorm + RoPE epilogue */
  ZI_KERNEL_ATTENTION = 2,      /* flash attention */
  ZI_KERNEL_GEMM_OUT = 3,       /* attention output projection */
  ZI_KERNEL_GEMM_FFN_UP = 4,    /* w1|w3 projection + SwiGLU epilogue */
  ZI_KERNEL_GEMM_FFN_DOWN = 5,  /* w2 projection */
  ZI_KERNEL_POST_NORM = 6,      /* post-norm + gated residual + next pre-norm */
  ZI_KERNEL_PRE_NORM = 7,       /* RMSNorm x (1 + scale) -> bf16 */
  ZI_KERNEL_ADALN = 8,          /* all adaLN projections */
  ZI_KERNEL_TIMESTEP = 9,       /* timestep sinusoid + MLP */
  ZI_KERNEL_ROPE = 10,          /* RoPE cos/sin table */
  ZI_KERNEL_POSITIONS = 11,     /* position ids */
  ZI_KERNEL_PATCHIFY = 12,      /* latent -> patch tokens */
  ZI_KERNEL_GEMM_EMBED = 13,    /* x_embedder / cap_embedder projection */
  ZI_KERNEL_GEMM_FINAL = 14,    /* final linear + unpatchify */
  ZI_KERNEL_EULER = 15,         /* Euler / CFG step */
  ZI_KERNEL_GEMM = 16,          /* zi_gemm_bf16 */
  ZI_KERNEL_TEXT_PAD = 17,      /* cap_pad_token into padded text rows */
  ZI_KERNEL_SPLIT_CLEAR = 18,   /* zero the GEMM split-tail counters (once per forward) */
  ZI_KERNEL_QUANTIZE = 19,      /* zi_quantize_rows_e4m3 */
  ZI_KERNEL_SELFTEST = 20,      /* zi_watchdog_selftest */
  ZI_KERNEL_EXP2_TEST = 21      /* zi_exp2_poly */
};

/* Start recording launch timings on this host thread: from the next kernel the
 * library enqueues, a timing event is recorded before the first kernel and after
 * every kernel (up to `capacity` kernels), on the launching stream.  Creates
 * capacity + 1 CUDA events (no device memory).  ZI_ERR_ARG if already started. */
ZI_API int zi_profile_begin(int capacity);

/* Stop recording: waits for the last recorded event, writes per-launch times in
 * milliseconds (time from the previous marker to this kernel's end marker) to
 * h_ms and zi_kernel_kind ids to h_kinds (up to `capacity` entries each; either
 * may be NULL), the number of launches to *h_count (-1 if more kernels ran than
 * the capacity given to zi_profile_begin), and destroys the events. */
ZI_API int zi_profile_end(float* h_ms, int* h_kinds, int capacity, int* h_count);

/* ---------------------------------------------------------------- device status */

/* Failure-detection self-test: enqueues one kernel whose single waiting thread
 * spins on an mbarrier that nothing completes, with the library's bounded wait
 * (here limit_us microseconds, 1 .. 2,000,000; else ZI_ERR_ARG).  When the
 * limit runs out the kernel records a timeout in the device error word (raw
 * code 6) and returns, so the context stays usable: zi_device_status() then
 * reports ZI_ERR_TIMEOUT, and until zi_clear_device_status() every pipeline
 * kernel of the library exits at once without touching memory. */
ZI_API int zi_watchdog_selftest(int limit_us, zi_stream_t stream);

/* Reads (synchronously) the device error word of the current device: ZI_OK, or
 * ZI_ERR_TIMEOUT if a kernel's bounded pipeline wait ran out since the last
 * zi_clear_device_status(); *h_code (may be NULL) receives the raw code. */
ZI_API int zi_device_status(int* h_code);

/* Clears the device error word (synchronously).  While it is set, every
 * pipeline kernel of the library exits at once without touching memory. */
ZI_API int zi_clear_device_status(void);

#ifdef __cplusplus
}
#endif

#endif /* ZIMAGE_DIT_H */
