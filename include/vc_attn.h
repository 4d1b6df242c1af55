/*
 * vc_attn.h - C ABI of libvcattn, VC-Attention FP8 for NVIDIA B200 (sm_100a).
 *
 * VC-Attention is a training-free, non-causal, quantized attention forward
 * pass for diffusion transformers. Sources (web pages, by title and section):
 *  [VCA]  "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58×
 *         sem retreinamento": "Por que a atenção é o gargalo" (low-bit tensor
 *         cores for QK^T and PV; Q/K smoothing is prior art), "V-Smooth:
 *         corrigindo outliers de valor" (Group, Demean, Restore), "ExpCast-FP8:
 *         eliminando o gargalo do softmax" (byte ~ 8*log2(p) + 56 by one FMA).
 *  [IP73] "VC-Attention et FLUX 3 accélèrent la génération d'images sur
 *         Blackwell", "Le compromis entre vitesse et fidélité" (repair budget
 *         rho = 0.005 for the tokens with the largest quantization error).
 *
 * Conventions for every call:
 *  - Tensors are dense, row-major, in device memory unless stated. Q, K, V
 *    and O are bf16 [B, H, N, d] with d = 128 (any other d is
 *    VC_ERR_UNSUPPORTED). Nb = ceil(N/128) blocks, Npad = 128*Nb.
 *  - The caller owns and allocates every buffer, including the workspace
 *    sized by vc_attn_workspace_bytes(); the library allocates nothing and
 *    keeps no state between calls (the per-device tensor-map encoder entry
 *    point is looked up once).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *    asynchronous on it; argument errors are detected on the host before any
 *    launch and nothing is launched then.
 *  - Device pointers must be 16-byte aligned (TMA); the workspace 256-byte
 *    aligned. B*H*Npad*d must be < 2^31.
 *  - Inputs containing NaN/Inf give undefined (but bounded-time) results.
 *  - Device-side waits are bounded; a wait that runs out sets a status word
 *    in the workspace, read back with vc_attn_device_status().
 */
#ifndef VC_ATTN_H
#define VC_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VC_OK = 0,
  VC_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or parameter */
  VC_ERR_UNSUPPORTED = 2, /* d != 128, device not compute capability 10.0 */
  VC_ERR_WORKSPACE = 3,   /* workspace smaller than vc_attn_workspace_bytes() */
  VC_ERR_CUDA = 4,        /* a CUDA runtime call failed */
  VC_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out */
} vc_status;

/* Method switches (vc_params.flags). */
#define VC_VSMOOTH 1u /* V-Smooth: k-means grouping + block demean/restore */
#define VC_REPAIR 2u  /* rho-repair of the worst-quantized value tokens */
#define VC_KSMOOTH 8u /* subtract the per-(b,h) channel mean of K */
/* vc_attn_cluster / vc_attn_cluster_noalloc only: start the Lloyd iterations
 * from the centroids passed in (the previous denoising step's) instead of the
 * tokens V[floor(j*N/k)]. Ignored by vc_attn_fwd, which clusters from scratch. */
#define VC_WARMSTART 16u
/* The NVFP4-residual variant ([VCA] "V-Smooth…", item Demean: the residual in
 * NVFP4 for the 4-bit kernel; "ExpCast-FP8…": ExpCast is 8-bit only). The V
 * residual is stored as E2M1 codes with an E4M3 scale per 16 consecutive
 * permuted tokens of a channel and a per-channel power-of-two global scale;
 * the probabilities come from an exp2 softmax, quantized to NVFP4 per 16 keys;
 * PV runs on the block-scaled FP4 tensor cores. QK^T stays FP8; the expcast
 * bias is not used. vc_attn_quant_v and vc_attn_fwd honour it. */
#define VC_VFMT_NVFP4 32u
/* The full 4-bit path ([VCA] "Por que a atenção é o gargalo": low-precision
 * tensor cores for both products; "Benchmarks": the 4-bit V-Smooth kernel
 * against SageAttention3): with VC_VFMT_NVFP4, Q and K' are NVFP4 too and
 * QK^T runs on the block-scaled FP4 tensor cores. Per 128-row block of Q
 * (original order) or K' (permuted order, K smoothing applied) a power-of-two
 * global scale g, the least with amax <= 2688 * g (1 for an all-zero block);
 * per row and 16 consecutive channels an E4M3 scale sf = E4M3(fp32(b / g) / 6)
 * of the block maximum b; codes E2M1(fp32(x / g) * fp32(1 / sf)) (0 where sf
 * is 0). The score scale is g_q * g_k * kappa. Without VC_VFMT_NVFP4 the
 * flag is invalid. vc_attn_quant_qk and vc_attn_fwd honour it. */
#define VC_QK_NVFP4 64u
/* The prologue of vc_attn_fwd (clustering when no permutation is passed,
 * Q/K smoothing and quantization, V demean + quantization, repair list and
 * deltas) as one cooperative persistent launch instead of one launch per
 * step: every block of the grid is resident, the steps follow each other
 * behind grid-wide barriers (bounded: a barrier that runs out sets
 * VC_ERR_TIMEOUT in the device status word). Bit-identical results. Applies
 * to the E4M3 path with k <= 8; otherwise the flag is ignored. vc_attn_fwd
 * honours it; its profile then reports the whole prologue as the first
 * phase. */
#define VC_FUSED_PROLOGUE 128u

typedef struct {
  int k;             /* k-means clusters, 1..64 (default 8) */
  int iters;         /* Lloyd iterations, 0..64 (default 3) */
  float rho;         /* repair budget, [0, 1) (default 0.005); R = ceil(rho*N) */
  float softmax_scale; /* 0 => 1/sqrt(d) */
  int expcast_bias;  /* C: the running row maximum maps to byte C, 8..126 (default 120) */
  unsigned flags;    /* VC_VSMOOTH | VC_REPAIR | VC_KSMOOTH (default), optionally VC_WARMSTART,
                        VC_VFMT_NVFP4, VC_QK_NVFP4 (with VC_VFMT_NVFP4), VC_FUSED_PROLOGUE */
} vc_params;

/* Fill the defaults listed above. */
void vc_params_default(vc_params *p);

/* Human-readable name of a status code (static string). */
const char *vc_status_str(vc_status s);

/* Bytes of workspace vc_attn_fwd / vc_attn_cluster / vc_attn_quant_v need for
 * this shape and these parameters (the largest of the three). 0 on bad args. */
size_t vc_attn_workspace_bytes(int B, int H, int N, int d, const vc_params *p);

/* Number of repair tokens per (b,h) for these parameters: ceil(rho*N) when
 * VC_REPAIR is set, else 0 (rho*N evaluated in double from the float rho). */
int vc_attn_repair_count(int N, const vc_params *p);

/*
 * V-Smooth Group ([VCA] "V-Smooth…", item Group): deterministic Lloyd k-means
 * over the value tokens of every (b,h), then a stable sort of token indices by
 * cluster label.
 *   V        bf16 [B,H,N,d]                       in
 *   perm     int32 [B,H,N] out: perm[p] = original index of the token at
 *            permuted position p (K and V are both read through it)
 *   centroids fp32 [B,H,k,d] out (final centroids), or NULL; in and out
 *            with VC_WARMSTART (then required: the starting centroids)
 * Init c_j = V[floor(j*N/k)] (or the given centroids with VC_WARMSTART, the
 * cross-step form of the pages' online grouping, which they run only in the
 * first quarter of the denoising steps); distances are fp32, accumulated by fma in
 * channel order; ties go to the lowest cluster; centroid = fp32(fp64 sum /
 * count); an empty cluster keeps its centroid; `iters` rounds, then a final
 * assignment. Bit-identical to the CPU oracle.
 */
vc_status vc_attn_cluster(const void *V, int B, int H, int N, int d, const vc_params *p, int32_t *perm,
                          float *centroids, void *ws, size_t ws_bytes, void *stream);

/*
 * vc_attn_cluster without a workspace. The pages have no counterpart: this
 * is a library convenience. It is for callers that cannot allocate device
 * memory where they cluster - for example a plugin inside a host framework
 * that owns every allocation and hands out no scratch, a deployment that
 * forbids cudaMalloc after start-up so that memory use stays fixed, or code
 * running where an allocation would synchronize the device. Such callers
 * still pass V (input) and perm and centroids (outputs, centroids not NULL);
 * the scratch (labels, k-means partial sums, completion counters) lives in a
 * fixed 32 MiB array in device memory that the library reserves on every
 * GPU that loads it, until the process exits.
 *   Output: identical to vc_attn_cluster with the same arguments.
 *   Limit: the scratch is 4 bytes per token (labels) plus the k-means
 *   partial sums (8*k*128 bytes per k-means block, about max(B*H, 444)
 *   blocks in all: 3.6 MB at k = 8 for up to 444 heads) and 256-byte-aligned
 *   counters. Shapes
 *   whose scratch exceeds 32 MiB (vc_attn_cluster_noalloc_max_bytes) return
 *   VC_ERR_WORKSPACE before any launch: about B*H*N <= 7.7 M tokens at k = 8
 *   while B*H <= 296 (each head past that adds 8 KB of partial sums); the
 *   720p video workload, 3.0 M tokens, fits.
 *   Set-up: the first call on each device looks up the array's device
 *   address (cudaGetSymbolAddress) with that device current; make that first
 *   call before any stream capture. cudaDeviceReset() ends the context that
 *   holds the array and makes that address stale: a process that resets a
 *   device must not call this entry point on it again. (A call that sees the
 *   context gone drops the cached address, so the next call looks it up
 *   again.)
 *   Calls allocate no memory (no cudaMalloc, cudaFree or allocating library
 *   routine). All calls share the one array and each call starts by clearing
 *   its counters; calls whose executions overlap on the GPU (other streams,
 *   other host threads) race on it and must be serialized by the caller.
 */
vc_status vc_attn_cluster_noalloc(const void *V, int B, int H, int N, int d, const vc_params *p, int32_t *perm,
                                  float *centroids, void *stream);

/* Size in bytes of the fixed scratch array behind vc_attn_cluster_noalloc. */
size_t vc_attn_cluster_noalloc_max_bytes(void);

/*
 * Q/K smoothing + 8-bit quantization (prior art named in [VCA] "Por que a
 * atenção é o gargalo"): K' = K - mean_n(K) per (b,h,channel) when
 * VC_KSMOOTH is set; Q (original order) and K' (rows read through perm) are
 * quantized per 128-row block to E4M3 with scale = amax/448.
 *   Q, K  bf16 [B,H,N,d] in;  perm int32 [B,H,N] in (NULL = identity)
 *   q8, k8 uint8 [B,H,Npad,d] out (E4M3 codes; padding rows are 0)
 *   sq, sk fp32 [B,H,Nb] out (block scales)
 * With VC_QK_NVFP4 (see there) the same buffers receive NVFP4 tile images
 * instead, one per 128-row block, 9216 bytes each at byte (b*H+h)*Nb*9216 +
 * t*9216 (the first 9/16 of the buffer): the E4M3 scales (byte 512*(j/4) +
 * 16*(r%32) + 4*(r/32) + j%4 for row r and 16-channel block j), then the E2M1
 * codes, rows of 64 bytes (channel 2i in the low nibble of byte i) in the
 * 64-byte swizzle of the V tile images; rows past N are 0. sq, sk receive the
 * power-of-two global scales g.
 */
vc_status vc_attn_quant_qk(const void *Q, const void *K, const int32_t *perm, int B, int H, int N, int d,
                           const vc_params *p, uint8_t *q8, float *sq, uint8_t *k8, float *sk, void *ws,
                           size_t ws_bytes, void *stream);

/*
 * V-Smooth Demean + residual quantization ([VCA] "V-Smooth…", item Demean)
 * and the rho-repair list ([IP73] "Le compromis…").
 *   V           bf16 [B,H,N,d] in;  perm int32 [B,H,N] in (NULL = identity)
 *   v8          uint8 [B,H,d,Npad] out: E4M3 residual codes, CHANNEL-MAJOR
 *               (v8[b,h,c,p] is channel c of the token at permuted position
 *               p); padding positions are 0
 *   v_scale     fp32 [B,H,d] out: per-channel power-of-two scale, the least
 *               2^e with max_p |r| <= 448 * 2^e (1 for an all-zero channel)
 *   v_mean      bf16 [B,H,Nb,d] out: block means (0 without VC_VSMOOTH)
 *   rep_idx     int32 [B,H,R] out: permuted positions of the R repaired
 *               tokens, ascending (R = vc_attn_repair_count); may be NULL if R=0
 *   rep_delta   bf16 [B,H,R,d] out: bf16(residual - dequantized code)
 * Blocks are 128 consecutive permuted positions (tail block: the rest);
 * mean = bf16(fp32(fp64 sum / count)); r = v - mean; code = E4M3(r * 2^-e);
 * token error = sum_c (r - value(code)*scale)^2 (fp32, fma in channel order);
 * the R largest errors are repaired (ties to the lowest position).
 * With VC_VFMT_NVFP4 the residual is NVFP4 instead:
 *   v8          holds B*H*Nb tile images of 9216 bytes (the buffer size is
 *               the same B*H*d*Npad bytes; the images fill the first 9/16):
 *               bytes [0,1024) the E4M3 block scales, byte 512*(j/4) +
 *               16*(c%32) + 4*(c/32) + j%4 for channel c and 16-token block
 *               j of the tile; bytes [1024,9216) the E2M1 codes, channel row c
 *               of 64 bytes (token 2i in the low nibble of byte i) with byte i
 *               of row c at 1024 + 512*(c/8) + 64*(c%8) + 16*((i/16) XOR
 *               ((c/2)%4)) + i%16 (the 64-byte swizzle of the tensor cores)
 *   v_scale     per-channel global scale g = 2^e, the least with
 *               max_p |r| <= 2688 * 2^e (2688 = 6 * 448)
 *   sf = E4M3(fp32(b * 2^-e) / 6) for the block maximum b = max |r|;
 *   code = E2M1(fp32(r * 2^-e) * fp32(1/sf)) (0 when sf is 0); token error
 *   and repair as above with value(code) * sf * g.
 */
vc_status vc_attn_quant_v(const void *V, const int32_t *perm, int B, int H, int N, int d, const vc_params *p,
                          uint8_t *v8, float *v_scale, void *v_mean, int32_t *rep_idx, void *rep_delta,
                          void *ws, size_t ws_bytes, void *stream);

/*
 * The VC-Attention FP8 forward: O = attention(Q, K, V) for every (b,h).
 *   Q, K, V  bf16 [B,H,N,d] in
 *   perm     int32 [B,H,N] in, or NULL: cluster now when VC_VSMOOTH is set
 *            (the pages run the grouping only in the first 25% of denoising
 *            steps and reuse the permutation after), identity otherwise
 *   O        bf16 [B,H,N,d] out, rows in the original query order
 * Steps: K smoothing + Q/K quantization; V demean + per-channel E4M3
 * residual + repair list; then one fused kernel per 128-query tile on the
 * tcgen05 tensor cores: S = Q8 K8^T (FP8, fp32 in TMEM); online row max in
 * "byte units" (8 * log2 of the probability) against the frame
 * F = 8*ceil(max/8); ExpCast: byte = RNE(fp32(acc*alpha + C - F)) clamped at
 * 0 - one fused multiply-add, no exponential; O += P V8 (FP8); the per-tile
 * row sum l_t of the decoded bytes comes out of the same MMA (a ones column),
 * and the block mean is restored as l_t * mean_t ([VCA] "V-Smooth…", item
 * Restore) on the tensor cores in bf16; repair adds p * delta for the listed
 * tokens; O = scale_c * acc / l.
 * Q/K quantization runs on an internal non-blocking stream of the library
 * (one per device, created on first use with three events), ordered by
 * events: when the call clusters, the K channel means and Q start with the
 * call (they do not depend on the permutation) and K' follows the
 * clustering; otherwise Q and K' are one launch. Either way it overlaps the
 * V passes; the call stays stream-ordered with respect to the caller's
 * stream and can be captured into a CUDA graph. Concurrent calls from
 * several host threads on one device serialize on that side stream (a
 * per-device lock is held while a call enqueues its work).
 * With VC_VFMT_NVFP4 (the 4-bit variant): the same frames, then per 16 keys
 * x = fma(acc, alpha/8, -F/8), p = 2^x, block scale sf = E4M3(448 * max p),
 * codes E2M1(p * fl(2688/sf)); O += P V4 on the block-scaled FP4 tensor cores
 * (kind::mxf4nvf4) with the row sums from the same product; repair uses
 * bf16(2^x' * 2688) with x' against the final frame.
 */
vc_status vc_attn_fwd(const void *Q, const void *K, const void *V, int B, int H, int N, int d,
                      const int32_t *perm, const vc_params *p, void *O, void *ws, size_t ws_bytes, void *stream);

/*
 * vc_attn_fwd from host memory: the same forward pass (clustering inside the
 * call), with Q, K, V read from host buffers and O written to a host buffer.
 * The (b,h) heads are split into `groups` runs of consecutive heads. Every step
 * of the method is per head, so the result is bit-identical to vc_attn_fwd.
 *
 * Per run, the call:
 *   1. copies the run's Q, K and V slices host -> device;
 *   2. runs the forward on that run;
 *   3. copies the run's O slice back device -> host.
 * The copies go on two non-blocking streams the library keeps per device
 * (created by the first call, with their events), so the copy-in of one run
 * and the copy-out of another overlap the computation of a third. Concurrent
 * calls from several host threads on one device serialize on them.
 *
 * Host buffers: hQ, hK, hV, hO, [B][H][N][d] bf16. They should be page-locked
 * (cudaHostAlloc or cudaHostRegister); pageable memory works but does not
 * overlap.
 * Device buffers: dQ, dK, dV, dO, each B*H*N*d bf16, owned by the caller and
 * used as staging.
 * Workspace: ws is a workspace for ONE run, i.e.
 *   vc_attn_workspace_bytes(1, ceil(B*H / groups), N, d, p).
 * groups: 1 .. B*H; it is clamped to B*H.
 *
 * Ordering: the call is asynchronous. Its work is ordered after earlier work on
 * `stream`, and later work on `stream` is ordered after its last copy.
 * Errors: as vc_attn_fwd, plus VC_ERR_INVALID_ARG for a null host or device
 * pointer or groups < 1.
 *
 * The pages give no host interface (the kernel is proprietary); this call is the
 * end-to-end form of vc_attn_fwd that the measurement uses.
 */
vc_status vc_attn_fwd_host(const void *hQ, const void *hK, const void *hV, int B, int H, int N, int d,
                           const vc_params *p, void *hO, void *dQ, void *dK, void *dV, void *dO, int groups,
                           void *ws, size_t ws_bytes, void *stream);

/*
 * In-library comparator: exact-softmax attention in BF16 on the tcgen05
 * tensor cores (bf16 operands, fp32 accumulation, fp32 exp2 softmax). The
 * pages measure VC-Attention against a BF16 FlashAttention-class kernel
 * ([IP73] intro: 1.46-1.59x over BF16 FlashAttention-4 on datacenter
 * Blackwell and Hopper; [VCA] "Benchmarks"); this is the library's own BF16
 * attention on the same tiling, for the same comparison on one GPU.
 *   Q, K, V  bf16 [B,H,N,d] in (d = 128), device pointers, 16-byte aligned
 *   O        bf16 [B,H,N,d] out, rows in query order
 *   softmax_scale 0 => 1/sqrt(d)
 * No workspace: a bounded device wait that runs out shows only as a wrong
 * result. Errors as vc_attn_fwd's argument and device checks.
 */
vc_status vc_attn_fwd_ref_bf16(const void *Q, const void *K, const void *V, int B, int H, int N, int d,
                               float softmax_scale, void *O, void *stream);

/*
 * ExpCast on the device, element-wise, exactly as the attention kernel
 * computes it ([VCA] "ExpCast-FP8…"): out[i] = clamp(RNE(fp32(acc[i]*alpha[i]
 * + c[i])), 0, ...) where the result must not exceed 126 (the kernel never
 * produces more than C). n must be even; element pairs (2j, 2j+1) must share
 * alpha and c (the kernel processes pairs). Device pointers.
 */
vc_status vc_attn_expcast(const float *acc, const float *alpha, const float *c, long long n, uint8_t *out,
                          void *stream);

/* Hardware E4M3 encoding (round to nearest even, saturating to +/-448) of n
 * floats, as the quantization kernels use it. n even. Device pointers. */
vc_status vc_attn_e4m3_encode(const float *x, long long n, uint8_t *out, void *stream);

/* Read (synchronously, on `stream`) and clear the device status word kept in
 * the workspace: VC_OK, or VC_ERR_TIMEOUT if a bounded device wait ran out.
 * Every call that takes a workspace clears the word when it starts, so the
 * word reports on the most recent such call. */
vc_status vc_attn_device_status(void *ws, void *stream);

/* Self test of the bounded device waits: launches one thread that waits on a
 * barrier nothing arrives at, giving up after `limit_cycles` SM clock cycles
 * (1 .. 2^32); it then records the timeout in the workspace status word the
 * way the attention kernels do. Afterwards vc_attn_device_status(ws) returns
 * VC_ERR_TIMEOUT. No GPU state is harmed; the kernel returns normally. */
vc_status vc_attn_wait_selftest(void *ws, long long limit_cycles, void *stream);

/* Opt-in phase timing for benchmarks (single-threaded use). While on, every
 * vc_attn_fwd records CUDA events on its stream around its phases, with no
 * host synchronization; the events (a ring of the last 64 calls) are created
 * once per device when profiling is first switched on, and switching it on
 * again restarts the count. vc_attn_profile_read() waits for the recorded
 * calls and writes their mean phase durations in milliseconds to ms[0..3]:
 * clustering (0 when a permutation was passed; Q quantization may run
 * beside it on the internal side stream); V quantization + repair selection
 * (on the caller's stream, while K' quantization runs on the side stream);
 * the further wait for Q/K quantization (0 when it finished first); and the
 * fused attention kernel. Returns
 * the number of values written (4), or 0 if nothing was recorded or
 * max_n < 4. */
vc_status vc_attn_profile(int on);
int vc_attn_profile_read(float *ms, int max_n);

/* Number of kernels this library has launched in this process (for the
 * bench's launch count). */
unsigned long long vc_attn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* VC_ATTN_H */
