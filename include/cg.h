/*
 * cg.h -- C ABI of libcg, a B200 (sm_100a) implementation of the Codec-Gauge
 * cache-coordinate codec round trip on KV tensors.
 *
 * Source method: "Codec-Gauge: Learning Compression-Friendly Gauges for
 * Transformer KV Caches" (arXiv 2607.20538).  A small orthogonal gauge
 * G = exp(A - A^T) per (layer, K/V, head, channel group) maps cached keys and
 * values into coordinates a fixed low-bit backend preserves better; it is
 * applied before quantization and inverted (G^T) before attention.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every pointer argument named *_dev is DEVICE memory owned by the
 *           caller; the library never allocates, frees or retains device
 *           memory between calls (a caller-sized workspace is passed where a
 *           kernel needs scratch).  Descriptors are HOST structs read during
 *           the call only.
 * Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *           work is enqueued asynchronously; nothing synchronizes the host.
 * Layout.   The KV cache is bf16 [L][2][B][H][T][d], row-major, s = 0 keys and
 *           s = 1 values, T the token capacity.  Gauges are fp32
 *           [L][2][H][R][g][g] with R = d / g, row-major, y_i = sum_j G[i][j] x_j
 *           for the g-vector x of one token in one channel group (shared over
 *           the batch).
 * Errors.   Argument errors (null or misaligned pointers, unsupported sizes,
 *           token ranges off the block grid) return CG_ERR_INVALID or
 *           CG_ERR_UNSUPPORTED before anything is enqueued, and leave every
 *           output untouched.  A failed launch returns CG_ERR_CUDA.  Kernels
 *           that wait on asynchronous copies bound every wait; a wait that runs
 *           out records a device status word that cg_sync_status() reports as
 *           CG_ERR_TIMEOUT.  Inputs must be finite: NaN or Inf values give
 *           unspecified codes (no fault).
 * Alignment. All device pointers must be 16-byte aligned.
 * Threads.  Calls are re-entrant; concurrent calls on different streams are
 *           independent (apart from the shared status word).
 */
#ifndef CG_H_
#define CG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CG_OK = 0,
  CG_ERR_INVALID = 1,     /* bad argument: null, misaligned, out of range   */
  CG_ERR_UNSUPPORTED = 2, /* valid request this build has no kernel for     */
  CG_ERR_CUDA = 3,        /* launch or runtime error                        */
  CG_ERR_TIMEOUT = 4,     /* a bounded device-side wait ran out             */
  CG_ERR_TOO_LARGE = 5,   /* request exceeds a fixed, built-in scratch size */
  CG_ERR_BOUND = 6        /* CG_ENGINE_CHAIN_TENSOR: a tensor-core value lay
                             farther from the fp32 chain than the error bound
                             its decisions assume (see cg_sync_status)      */
} cg_status;

typedef enum {
  CG_QUANT_BLOCK_UNIFORM = 0, /* one min/max range per T_b x W block          */
  CG_QUANT_KIVI = 1           /* keys per channel, values per token           */
} cg_quant_mode;

/* Which gauge contraction feeds the quantizer in cg_encode.  The codes, steps
 * and zero points are always the quantizer's exact fp32 result for the gauged
 * values that engine produced (returned through the optional gauged output);
 * the engines differ in how those gauged values are defined.  Decode does not
 * depend on the engine. */
typedef enum {
  CG_ENGINE_AUTO = 0,         /* the fastest kernel for the request:
                                 g = 16 with W = 16, and KIVI-style with g = 16
                                 (d 64 or 128): tensor-core contraction with G
                                 split into two bf16 terms (within about 2^-17
                                 sum_j |G_ij x_j| of G x);
                                 g = d: tensor cores with G rounded to bf16;
                                 otherwise the fp32 FMA chain */
  CG_ENGINE_CUDA_CORES = 1,   /* the fp32 FMA chain on CUDA cores (g < d only):
                                 y_i = fl32(G_ij x_j + acc), j = 0..g-1 from +0,
                                 bit-reproducible on any device */
  CG_ENGINE_CHAIN_TENSOR = 2  /* the same codes as CG_ENGINE_CUDA_CORES, with the
                                 contraction on the 5th-generation tensor cores
                                 (g = 16, d = 128, W = 16 only): G split exactly
                                 into three bf16 terms, and the chain re-evaluated
                                 wherever the tensor-core value could change a
                                 decision (needs G orthogonal to 2^-12, checked
                                 per head slice; else the chain throughout).
                                 The decisions assume a tensor-core accumulation
                                 error of at most 2^-20 sum_j |G_ij x_j|; every
                                 value the chain re-evaluates is checked against
                                 that bound, and a value outside it sets a status
                                 bit that cg_sync_status reports as CG_ERR_BOUND */
} cg_engine;

/* Shape of a KV cache: K_l, V_l in R^{B x H x T x d} for l = 1..L
 * (Codec-Gauge, Problem statement and overview).  `tokens` is the capacity T
 * of the buffer; encode/decode take a token range inside it. */
typedef struct {
  int32_t layers;  /* L */
  int32_t batch;   /* B */
  int32_t heads;   /* H (KV heads) */
  int32_t tokens;  /* T (capacity), a multiple of 32 */
  int32_t d_head;  /* d: 64 or 128 */
} cg_kv_desc;

/* Codec settings.
 *   g           gauge group size: 8, 16, 32 (grouped) or d_head (full head)
 *               (Codec-Gauge, Method: g = 8, 16, 32 and full-head gauges).
 *   bits        bits per value: 2, 3, 4, 6 or 8 (Experimental setup).
 *   tb          token block T_b of the block-uniform ranges: 16.
 *   range_cols  W, channels per block-uniform range: g (default) or d_head
 *               (the page's "one range per T_b x d_l block").
 *   mode        cg_quant_mode.
 *   kivi_key_tokens, kivi_val_channels: KIVI group sizes, both 32.
 *   engine      cg_engine (encode only; decode ignores it).
 */
typedef struct {
  int32_t g;
  int32_t bits;
  int32_t tb;
  int32_t range_cols;
  int32_t mode;
  int32_t kivi_key_tokens;
  int32_t kivi_val_channels;
  int32_t engine;
} cg_codec_desc;

/* Buffer sizes of an encoded cache (whole capacity T).  The zero-point and
 * scale arrays are fp16 with scale_count entries each, so the actual
 * bits/value is 8 (code_bytes + 4 scale_count) / N_KV with
 * N_KV = sum_l 2 B H T d (Codec-Gauge, Problem statement; Experimental setup:
 * actual bits/value computed from measured bytes). */
typedef struct {
  uint64_t code_bytes;
  uint64_t scale_count;
} cg_sizes;

/* Spectral-statistics settings (Codec-Gauge, Method: T_b = 16,
 * lambda_f = 1.0, lambda_r = 0.02, tau = 0.04 for every checkpoint). */
typedef struct {
  int32_t tb;        /* token block of the DCT: 16 */
  int32_t g;         /* group size of G when a gauge is fused, else 0 */
  int32_t x_is_fp32; /* 1: x is fp32, 0: x is bf16 */
  float lambda_f;
  float lambda_r;
  float tau;
} cg_stats_desc;

/* Host only.  Fills *out with the exact byte / entry counts of the encoded
 * buffers for `kv` and `codec`; validates both descriptors.
 *   block-uniform: code_bytes = L 2 B H T d bits / 8,
 *                  scale_count = L 2 B H (T / tb) (d / W)
 *   KIVI:          code_bytes as above, scale_count = L 2 B H T d / 32 */
cg_status cg_sizes_for(const cg_kv_desc* kv, const cg_codec_desc* codec, cg_sizes* out);

/* G = exp(A - A^T) for n_mats independent g x g matrices
 * (Codec-Gauge, Method: gauge parameterization; the displayed equation is
 * missing from the page, which names exp(.) and the skew matrix A - A^T).
 *   A_dev, G_dev : fp32 [n_mats][g][g], row-major, may not alias.
 *   g            : 2 .. 128.
 * Scaling and squaring with a degree-14 Taylor core, in fp64 (above g = 64 the
 * scaled skew matrix is held in fp32), rounded once to fp32: G is within about
 * 1e-7 of exp(A - A^T) and orthogonal to about 1e-6.  One thread block per
 * matrix. */
cg_status cg_gauge_build(const float* A_dev, float* G_dev, int32_t n_mats, int32_t g, void* stream);

/* AdamW hyperparameters (Loshchilov & Hutter 2019, decoupled weight decay).
 * The pages name AdamW without its settings; torch's defaults are the reading
 * taken: lr 1e-3, betas (0.9, 0.999), eps 1e-8, weight decay 0.01. */
typedef struct {
  float lr;
  float beta1;
  float beta2;
  float eps;
  float weight_decay;
} cg_adamw_desc;

/* dL/dA from dL/dG for G = exp(A - A^T), for n_mats independent g x g matrices
 * (Codec-Gauge, Method: gauge parameterization and gauge training, where the
 * objective is optimized through exp).  dS = L_exp(S^T, dG), the adjoint of the
 * Frechet derivative, is the upper-right g x g block of
 * exp([[S^T, dG], [0, S^T]]) (Van Loan 1978; Higham 2008, section 10.6), and
 * dA = dS - dS^T.  One thread block per matrix, fp64 internally.
 *   A_dev, dG_dev (input), dA_dev (output): fp32 [n_mats][g][g], row-major;
 *   dA_dev may alias neither input.
 *   g: 2 .. 32 (CG_ERR_UNSUPPORTED above 32). */
cg_status cg_gauge_grad(const float* A_dev, const float* dG_dev, float* dA_dev, int32_t n_mats, int32_t g,
                        void* stream);

/* One AdamW step on n fp32 parameters in place (Codec-Gauge, Method: the gauge
 * is optimized with AdamW).  With t = step (1-based):
 *   m = b1 m + (1 - b1) grad,  v = b2 v + (1 - b2) grad^2,
 *   param -= lr (m / (1 - b1^t) / (sqrt(v / (1 - b2^t)) + eps) + wd param).
 *   param_dev, m_dev, v_dev: fp32 [n] (updated); grad_dev: fp32 [n] (input).
 *   m and v start at zero before step 1. */
cg_status cg_adamw_step(float* param_dev, const float* grad_dev, float* m_dev, float* v_dev, int64_t n,
                        const cg_adamw_desc* hp, int32_t step, void* stream);

/* Uncentered second-moment (Gram) matrices of every channel group
 * (Codec-Gauge, Experimental setup: the PCA/KLT control uses the uncentered
 * second-moment eigenbasis at the layer, K/V, head and group granularity):
 *   gram[l][s][h][r] = sum over b and t in [t0, t0 + nt) of x x^T, x the g-vector
 *   of group r of token t.
 *   kv_dev    bf16 [L][2][B][H][T][d] (input)
 *   gram_dev  fp64 [L][2][H][d/g][g][g] (output, every entry written)
 *   g: 8, 16 or 32; any t0 and nt inside [0, T].
 * Sums run in fp64 in a fixed order (one thread block per gauge set). */
cg_status cg_group_gram(const cg_kv_desc* kv, int32_t g, const void* kv_dev, int32_t t0, int32_t nt, double* gram_dev,
                        void* stream);

/* Fused gauge + quantize + pack for tokens [t0, t0 + nt) of every
 * (layer, K/V, batch, head)
 * (Codec-Gauge, Figure 1 / Backend compatibility: the gauge is applied at the
 * KV tensor interface before quantization; Experimental setup: block-uniform
 * and KIVI-style backends).
 *   kv_dev      bf16 [L][2][B][H][T][d]                         (input)
 *   G_dev       fp32 [L][2][H][d/g][g][g]                        (input)
 *   codes_dev   uint8, cg_sizes.code_bytes for the whole capacity (output)
 *   scales_dev, zeros_dev  fp16, cg_sizes.scale_count each       (output)
 *   gauged_dev  optional fp32 [L][2][B][H][T][d]: the gauged values the
 *               quantizer saw (NULL to skip; costs 4 B/value of traffic)
 * Only the blocks covering [t0, t0 + nt) are written.  t0 and nt must be
 * multiples of tb (block-uniform) or of 32 (KIVI).
 * Block-uniform layout: codes [L][2][B][H][T/tb][d/W][tb*W*bits/8], element
 * i = t_local*W + c_local of a block holding bits [i*bits, i*bits + bits) of a
 * little-endian bit stream; scales / zeros [L][2][B][H][T/tb][d/W].
 * KIVI layout: keys (s = 0) codes [..][T/32][d][32*bits/8] (token-ascending),
 * values (s = 1) codes [..][T][d/32][32*bits/8] (channel-ascending); scales /
 * zeros [..][T/32][d] and [..][T][d/32].
 * Per range: z = fp16(min), s = fp16(fl32(fl32(max - min) / (2^b - 1))),
 * q = clamp(rne(fl32(fl32(y - z) * fl32(1/s))), 0, 2^b - 1), q = 0 if s = 0.
 * Gauged values: see cg_engine.  Whatever the engine, the codes, steps and
 * zero points equal the quantizer above applied to the gauged values the
 * engine produced (bit for bit), and a zero block minimum or maximum is taken
 * as +0.  With CG_ENGINE_CHAIN_TENSOR the gauged output holds the values
 * actually quantized: within 2^-16 max|y| of the 16 x 16 block of the chain
 * and equal to it wherever the chain was evaluated, while the codes are the
 * chain's. */
cg_status cg_encode(const cg_kv_desc* kv, const cg_codec_desc* codec,
                    const void* kv_dev, const float* G_dev, int32_t t0, int32_t nt,
                    uint8_t* codes_dev, void* scales_dev, void* zeros_dev,
                    float* gauged_dev, void* stream);

/* Fused unpack + dequantize + inverse gauge for tokens [t0, t0 + nt)
 * (Codec-Gauge, Figure 1: the inverse gauge restores the KV state before
 * attention; Method: explicit key/value recovery, charged in timing).
 *   x_hat = G^T (s q + z) per token and group, written as bf16 (RNE) into
 *   kv_out_dev [L][2][B][H][T][d] (other tokens untouched).
 * Buffers and layouts as in cg_encode.  G for g = d is rounded to bf16. */
cg_status cg_decode(const cg_kv_desc* kv, const cg_codec_desc* codec,
                    const uint8_t* codes_dev, const void* scales_dev, const void* zeros_dev,
                    const float* G_dev, int32_t t0, int32_t nt, void* kv_out_dev, void* stream);

/* Workspace bytes cg_roundtrip_host needs: four layer-sized bf16 buffers,
 * 4 * 2 B H T d * 2 bytes (host only). */
cg_status cg_roundtrip_workspace_size(const cg_kv_desc* kv, uint64_t* bytes);

/* cg_encode followed by cg_decode of the whole cache, with the cache and the
 * decoded result in HOST memory (Codec-Gauge, Method: the codec round trip,
 * with the recovery charged in timing).  The work is cut into layers: the copy
 * of layer l + 1 to the device, the encode and decode of layer l and the copy
 * of layer l - 1 back to the host run at the same time, on three internal
 * non-blocking streams of the current device (created on first use and kept
 * for the life of the process), so the two PCIe directions overlap each other
 * and the kernels.
 *   kv_host     bf16 [L][2][B][H][T][d] in host memory (input; page-locked
 *               memory is needed for the copies to overlap)
 *   G_dev, codes_dev, scales_dev, zeros_dev: as in cg_encode (the codes of the
 *               whole cache are written, as by cg_encode over [0, T))
 *   out_host    bf16 [L][2][B][H][T][d] in host memory (output: the decoded
 *               cache, as cg_decode writes it)
 *   workspace_dev / workspace_bytes: at least cg_roundtrip_workspace_size().
 * The call is ordered after earlier work on `stream`, and later work on
 * `stream` is ordered after all of it; the host buffers must stay valid and
 * unchanged until then.  Concurrent calls on one device share the internal
 * streams (they stay correct, each with its own workspace, but queue behind
 * one another).  Argument errors as in cg_encode; CG_ERR_UNSUPPORTED
 * when one layer's codes, steps or zero points are not a multiple of 16 bytes
 * (the per-layer pointers must stay aligned). */
cg_status cg_roundtrip_host(const cg_kv_desc* kv, const cg_codec_desc* codec, const void* kv_host,
                            const float* G_dev, uint8_t* codes_dev, void* scales_dev, void* zeros_dev,
                            void* out_host, void* workspace_dev, uint64_t workspace_bytes, void* stream);

/* Decode-step attention settings.
 *   q_heads   query heads Hq, a multiple of the cache's KV heads H with
 *             Hq / H in {1, 2, 4, 8}; query head j uses KV head j / (Hq / H)
 *             (grouped-query attention).
 *   n_tokens  attend to cached tokens [0, n_tokens): a multiple of 16 in [16, T].
 *   layer0, n_layers  the layers [layer0, layer0 + n_layers) of this call.
 *   scale     score scale, usually 1 / sqrt(d_head). */
typedef struct {
  int32_t q_heads;
  int32_t n_tokens;
  int32_t layer0;
  int32_t n_layers;
  float scale;
} cg_attn_desc;

/* Workspace bytes cg_decode_attention needs (host only). */
cg_status cg_decode_attention_workspace_size(const cg_kv_desc* kv, const cg_attn_desc* at, uint64_t* bytes);

/* One decode step of attention read directly from the encoded cache, the
 * inverse gauge included (Codec-Gauge, Figure 1 / Backend compatibility: keys
 * and values are restored with G^T before attention).  For every layer l of
 * the call, batch b and query head j (KV head h = j / (Hq / H)):
 *   out = sum_t softmax_t(scale q . k_t) v_t,  t in [0, n_tokens),
 *   k_t = G_K^T (s q_t + z), v_t = G_V^T (s q_t + z) per 16-channel group,
 * computed as (G_K q) . y_K,t and G_V^T (sum_t p_t y_V,t): the gauge is applied
 * to the query and the output instead of every cached token (the same result).
 *   codec       block-uniform, g = 16, 16 x 16 ranges (range_cols = 16), any
 *               bits; d_head 64 or 128.
 *   q_dev       bf16 [n_layers][B][Hq][d] (input)
 *   codes_dev, scales_dev, zeros_dev, G_dev: the whole encoded cache, as
 *               cg_encode writes it and cg_decode reads it
 *   out_dev     fp32 [n_layers][B][Hq][d] (output)
 *   workspace_dev / workspace_bytes: at least
 *               cg_decode_attention_workspace_size() (per-chunk partials).
 * Scores and sums are fp32; softmax uses the max-shifted exponential. */
cg_status cg_decode_attention(const cg_kv_desc* kv, const cg_codec_desc* codec, const cg_attn_desc* at,
                              const void* q_dev, const uint8_t* codes_dev, const void* scales_dev,
                              const void* zeros_dev, const float* G_dev, float* out_dev, void* workspace_dev,
                              uint64_t workspace_bytes, void* stream);

/* Workspace bytes cg_spectral_stats needs for this shape (host only). */
cg_status cg_spectral_workspace_size(const cg_kv_desc* kv, const cg_stats_desc* st,
                                     int32_t want_grad, uint64_t* bytes);

/* Gauge-training statistics (Codec-Gauge, Method: frequency-distribution
 * objective).  Every T_b x d token-channel block of X' = G X (or of x itself
 * when G_dev is NULL) gets a 2-D orthonormal DCT-II U = C_Tb X' C_d^T; per
 * block
 *   L_freq = sum r_uv U_uv^2 / sum U_uv^2  (0 for an all-zero block),
 *   r_uv = sqrt((u/(T_b-1))^2 + (v/(d-1))^2) / sqrt(2),
 *   L_rate = mean log(1 + |U_uv| / tau)    (assumed form: the page's equation
 *                                           is truncated),
 * and L = lambda_f mean(L_freq) + lambda_r mean(L_rate).
 *   x_dev        bf16 or fp32 [L][2][B][H][T][d]
 *   G_dev        fp32 [L][2][H][d/g][g][g] or NULL (x already gauged)
 *   lfreq_dev, lrate_dev  fp32 [L][2][B][H][T/tb]              (output)
 *   totals_dev   fp64 [4]: sum L_freq, sum L_rate, n_blocks, L  (output)
 *   dG_dev       fp32 [L][2][H][d/g][g][g] = dL/dG, or NULL; requires G_dev
 *   workspace_dev / workspace_bytes: at least cg_spectral_workspace_size().
 * Shapes: d_head 64 or 128, T a multiple of 32 (tb = 16, g = 16 or no gauge);
 * d_head = 128 with T a multiple of 128 runs on the tensor cores, every other
 * shape on CUDA cores.  Reductions run in a fixed order: results are
 * deterministic for a given shape. */
cg_status cg_spectral_stats(const cg_kv_desc* kv, const cg_stats_desc* st,
                            const void* x_dev, const float* G_dev,
                            float* lfreq_dev, float* lrate_dev, double* totals_dev,
                            float* dG_dev, void* workspace_dev, uint64_t workspace_bytes,
                            void* stream);

/* cg_spectral_stats for callers that cannot allocate device memory.
 *
 * No counterpart in the paper: this is a deployment variant of the library.
 * Some callers are not allowed to allocate: code running inside a host
 * framework that hands out only pre-planned buffers (serving engines with a
 * fixed memory plan, plug-ins, real-time loops where cudaMalloc's implicit
 * synchronization is not acceptable) cannot create the workspace that
 * cg_spectral_stats needs for its dL/dG partials.  This entry point takes the
 * same arguments minus the workspace and uses a scratch array compiled into
 * the library instead (8 MiB per GPU, reserved on every GPU that loads the
 * library until the process exits).  It allocates nothing.
 *   Limit: the dG partials, d_head * 16 fp32 per work unit (two units per head
 *   slice at d_head = 128 with T a multiple of 256, one otherwise), must fit
 *   the 8 MiB array, i.e. L * 2 * B * H <= 512 at d_head = 128 (1024 when T is
 *   an odd multiple of 128 or not one of 128) and <= 2048 at d_head = 64, when
 *   dG_dev is given; larger requests return CG_ERR_TOO_LARGE before anything is
 *   enqueued.  Without dG_dev no scratch is used and there is no limit.
 *   Set-up: the first call on a device looks up the scratch array's device
 *   address (cudaGetSymbolAddress) with that device current; make that first
 *   call before any stream capture.
 *   Sharing: all calls on a device share the one scratch array.  Each call
 *   writes every scratch byte it later reads, so nothing needs clearing, but
 *   calls whose work overlaps on the GPU (different streams, no ordering) race
 *   on it and must be serialized by the caller.
 * Results, layouts and errors are otherwise those of cg_spectral_stats. */
cg_status cg_spectral_stats_noalloc(const cg_kv_desc* kv, const cg_stats_desc* st,
                                    const void* x_dev, const float* G_dev,
                                    float* lfreq_dev, float* lrate_dev, double* totals_dev,
                                    float* dG_dev, void* stream);

/* Self-test of the failure reporting (no counterpart in the paper: library
 * diagnostics).  Enqueues one small kernel that waits, with the library's own
 * bounded mbarrier wait and a limit of limit_ns nanoseconds (1 .. 2e9), on a
 * barrier that nothing ever completes.  The wait gives up after the limit, the
 * kernel writes 0 to *result_dev (1 would mean the wait completed) and ends
 * normally, and the next cg_sync_status() reports CG_ERR_TIMEOUT.  Nothing
 * faults or hangs; the device stays usable.
 *   result_dev  device uint32 (output).
 * Returns CG_ERR_INVALID for a limit out of range or a null pointer. */
cg_status cg_selftest_wait_timeout(int64_t limit_ns, uint32_t* result_dev, void* stream);

/* Synchronizes `stream`, then reports (and clears) the device status word:
 * CG_ERR_TIMEOUT if a bounded wait ran out since the last check, else
 * CG_ERR_BOUND if the chain-exact tensor-core encoder met a tensor-core value
 * outside its assumed error bound since the last check, CG_ERR_CUDA on a
 * pending CUDA error, else CG_OK. */
cg_status cg_sync_status(void* stream);

/* Name and description of the CUDA error behind the last CG_ERR_CUDA returned
 * on the calling host thread ("" if none).  The string is static. */
const char* cg_last_cuda_error(void);

/* Static, human-readable name of a status code. */
const char* cg_status_string(cg_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t cg_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CG_H_ */
