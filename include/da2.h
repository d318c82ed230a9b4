/*
 * da2.h -- C ABI of the DraftAttention2 hot path on NVIDIA B200 (sm_100a).
 *
 * Low-resolution-guided, block-sparse, mixed-precision self-attention over
 * spatiotemporal video-DiT tokens:
 *
 *   da2_prepare       fused operand preparation: per-frame 2D average- and max-pooled
 *                     draft Q/K, window-contiguous token permutation, FP8-E4M3 and
 *                     4-bit (E2M1, one E4M3 scale per 16 elements) copies of Q/K/V.
 *   da2_draft_select  low-resolution draft attention maps (avg- and max-pooled) combined
 *                     into a block-importance score, and the shared per-(head, query
 *                     block) ranking into FP8 / FP4 / skip under the budgets.
 *   da2_attention     one attention kernel with an FP8 phase and an FP4 phase that share
 *                     the online-softmax running max / sum and the fp32 accumulator; its
 *                     epilogue writes bf16 output back in the original token order.
 *
 * Sources: "DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-
 * Precision Attention" (arXiv 2609.32628), Abstract -- pooled draft Q/K, shared ranking
 * into higher / lower precision / skip under budgets, fused operand preparation, one
 * attention kernel with precision-specific phases sharing data movement, softmax
 * statistics and output accumulation. "DraftAttention: Fast Video Diffusion via
 * Low-Resolution Attention Guidance" (arXiv 2505.14708), Abstract -- per-frame
 * downsampling into draft Q/K, reorder before and restore after the sparse attention.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Inputs q, k, v and the output are bf16 [B, H, T, d] (or [B, T, H, d] with
 *    DA2_FLAG_LAYOUT_BTHD), d contiguous, with frame-major token order
 *    t = f*Hf*Wf + y*Wf + x.
 *  - Window (ph, pw) tiles each frame; edge windows are padded. Blocks n = f*ny*nx +
 *    (y/ph)*nx + (x/pw), slot s = (y%ph)*pw + (x%pw), ny = ceil(Hf/ph), nx = ceil(Wf/pw),
 *    N = F*ny*nx blocks of bs = ph*pw slots; padded slots hold zeros and padded keys are
 *    masked out of the attention.
 *  - Budgets: the shared ranking of each query block's KV blocks is cut three times,
 *    each cut rounded half up: c8 = floor((pct_fp8*N + 50)/100), c8m = floor(((pct_fp8 +
 *    pct_mix)*N + 50)/100), ck = floor(((pct_fp8 + pct_mix + pct_fp4)*N + 50)/100). The top
 *    n8 = c8 blocks are FP8, the next nm = c8m - c8 mixed (E4M3 Q K^T, E2M1 P V), the next
 *    n4 = ck - c8m FP4; the rest are skipped.
 *  - Memory ownership: the caller allocates q, k, v, out and the workspace (device memory,
 *    size from da2_workspace_size); the library allocates no device memory and keeps no
 *    state (da2_forward_host creates and destroys three streams and a few events per call;
 *    da2_forward_noalloc uses a static device array of the library image).
 *  - Every call is asynchronous on `stream` (0 = legacy default stream) except the ones
 *    documented as synchronising. Argument errors are returned before anything is
 *    enqueued; a failed CUDA call or launch returns DA2_ERR_CUDA, and da2_last_cuda_error
 *    then gives its cudaError_t.
 *  - Supported: d in {64, 128}; any window with bs = ph*pw in {32, 64, 128}; N <= 4096;
 *    B*H <= 65535 (DA2_ERR_UNSUPPORTED otherwise); 0 <= pct_fp8, pct_mix, pct_fp4 and
 *    pct_fp8 + pct_mix + pct_fp4 <= 100 (DA2_ERR_INVALID_ARG otherwise). Tensor pointers must be 16-byte
 *    aligned and the workspace 256-byte aligned (DA2_ERR_ALIGNMENT otherwise).
 */
#ifndef DA2_H
#define DA2_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* One attention call's shape, window and budgets. */
typedef struct da2_config {
  int B, H, d;          /* batch, heads, head dim (64 or 128) */
  int F, Hf, Wf;        /* latent frames, token rows and token columns per frame */
  int ph, pw;           /* pooling window rows x columns; block size bs = ph*pw */
  int pct_fp8, pct_fp4; /* percent of KV blocks kept at FP8 / FP4; the rest is skipped */
  float sm_scale;       /* softmax scale; 0 selects 1/sqrt(d) */
  int flags;            /* DA2_FLAG_* bits */
  int pct_mix;          /* percent of KV blocks in the mixed class (E4M3 scores, E2M1 P V),
                           ranked between FP8 and FP4; 0 gives the two-class path */
  float adapt_tau;      /* > 0: error-bound-driven FP4 budget. Per query block, the KV blocks
                           ranked after the fixed budgets join FP4, in rank order, while their
                           draft score (estimated attention mass) is >= adapt_tau, up to
                           pct_fp4_max percent FP4 blocks; 0 turns it off */
  int pct_fp4_max;      /* the FP4 cap of the adaptive budget (>= pct_fp4) */
} da2_config;

enum {
  /* da2_draft_select also writes its fp32 block-importance scores to the workspace
     (scores region, [B*H][N][N]); the workspace then grows by 4*B*H*N*N bytes. */
  DA2_FLAG_EXPORT_SCORES = 1,
  /* Drop the ln(valid tokens) term of the draft logits (the maps then rank by average
     token affinity instead of block mass). */
  DA2_FLAG_NO_MASS_CORRECTION = 2,
  /* q, k, v and out are token-major, bf16 [B,T,H,d] (the heads of one token adjacent, as
     a fused QKV projection usually leaves them) instead of [B,H,T,d]; read and written in
     place, results identical. da2_forward_host then runs unpipelined. (The pages fix no
     tensor layout.) */
  DA2_FLAG_LAYOUT_BTHD = 4,
  /* Debug aid: every workspace region is followed by a 256-byte guard (the workspace grows
     accordingly; da2_workspace_size and da2_workspace_views account for it). da2_prepare
     fills the guards with 0xA5 bytes and every stage call checks them after its kernels: a
     changed guard byte sets bit 4 of the workspace error word (DA2_ERR_TIMEOUT from
     da2_get_error). Costs two small launches per stage; off in normal use. */
  DA2_FLAG_DEBUG_CANARY = 8,
  /* Test hook for the failure path, never needed in use: da2_attention's copy engine
     withholds its first K/V tile, so a bounded device wait must run out. Every bounded
     wait's limit drops from 2 s to 50 ms; the launch sets the workspace error word, stops
     issuing, waits for its copies and tensor-core work in flight, frees its tensor memory
     and ends (about 0.1 s); da2_get_error then returns DA2_ERR_TIMEOUT and the output is
     undefined. */
  DA2_FLAG_TEST_STALL = 256
};

typedef enum da2_status {
  DA2_OK = 0,
  DA2_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, budgets out of range */
  DA2_ERR_UNSUPPORTED = 2,  /* d, bs, N or B*H outside the supported set */
  DA2_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
  DA2_ERR_WORKSPACE = 4,    /* ws_bytes smaller than da2_workspace_size */
  DA2_ERR_CUDA = 5,         /* a CUDA call or launch failed */
  DA2_ERR_TIMEOUT = 6,      /* the device error word is set (a bounded wait ran out, a bad
                               index, or an overwritten guard region) */
  DA2_ERR_SCRATCH_TOO_SMALL = 7 /* da2_forward_noalloc: the configuration's workspace does
                                   not fit the library's built-in 64 MiB device scratch */
} da2_status;

/* Byte offsets of the workspace regions (from the workspace base) and the geometry.
   Tile layouts (all per (b*H + h) then per block, each block tile contiguous):
     q8, k8   E4M3 [BH][N][tile8_qk]: bs rows (tokens) x d bytes in the tensor-core
              K-major core-matrix layout: byte (r, c) at (r/8)*(8*d) + (c/16)*128 +
              (r%8)*16 + c%16.
     q4, k4   E2M1 [BH][N][tile4_qk]: bs rows x d/2 bytes, element c in byte c/2 (even
              c in the low nibble), byte (r, b) at (r/8)*(4*d) + (b/16)*128 + (r%8)*16 +
              b%16.
     v8       E4M3 transposed [BH][N][tile8_v]: d rows (channels) x bs bytes (slots):
              byte (c, s) at (c/8)*(8*bs) + (s/16)*128 + (c%8)*16 + s%16.
     v4       E2M1 transposed [BH][N][tile4_v]: d rows x kv4/2 bytes, kv4 = max(bs, 64)
              (slots >= bs are zero codes): byte (c, b) at (c/8)*(4*kv4) + (b/16)*128 +
              (c%8)*16 + b%16.
     sfq4, sfk4  E4M3 group scales of q4/k4, [BH][N][sf_qk]: d/64 atoms of 512 bytes;
              atom kb holds rows 0..127 (rows >= bs zero) x 4 scales (channel groups
              4kb..4kb+3): byte (r, j) at kb*512 + (r%32)*16 + (r/32)*4 + j.
     sfv4     E4M3 group scales of v4, [BH][N][sf_v]: kv4/64 atoms; rows = channels
              (rows >= d zero), scales = slot groups: byte (c, j) at kb*512 + (c%32)*16 +
              (c/32)*4 + j for slot group 4kb + j (groups past bs are zero).
     sq, sk   fp32 [BH][N]   dequantisation scale of a Q / K block (block amax / 448).
     sv       fp32 [BH][d]   dequantisation scale of a V channel (channel amax / 448).
     vamax    fp32 [BH][d]   V channel amax (written by da2_prepare).
     qavg, qmax, kavg, kmax  fp32 [BH][N][d] pooled draft Q / K.
     tags     u8 [BH][N][N]  0 skip, 1 FP4, 2 FP8, 3 mixed for (query block, KV block).
     list8    i16 [BH][N][n8s], list4 i16 [BH][N][n4s], listm i16 [BH][N][nms]: kept KV
              blocks of each class per query block in ascending block order (n8s =
              max(n8,1), n4s = max(n4max,1), nms = max(nm,1)); with the adaptive budget a
              row's FP4 list holds its n4 .. n4max blocks followed by -1 entries.
     scores   fp32 [BH][N][N] (only with DA2_FLAG_EXPORT_SCORES, else size 0).
     dlog     fp32 [BH][N][2][np] the two draft logit rows (average map, max map) of every
              query block, written and read by da2_draft_select (scratch; size 0 when
              N > 1024).
     qt, kt   the pooled Q and K of qavg/qmax and kavg/kmax again, each value split into a
              tf32 high part and its fp32 remainder and laid out as the draft MMAs' operands:
              per (b, h), 128-block tile, map (average, max) and 16-channel chunk, an 8 KB hi
              part then an 8 KB lo part of 128 rows x 16 channels in the K-major core-matrix
              layout (written by da2_prepare, read by da2_draft_select; size 0 when N > 1024).
     err      u32 device error word (0 = no error): bit 1 a bounded wait ran out, bit 2 an
              index or count of the selection was out of range, bit 4 a guard region of
              DA2_FLAG_DEBUG_CANARY was overwritten.
   With DA2_FLAG_DEBUG_CANARY a 256-byte guard follows every region above.
   A DA2_DEBUG build of the library (libda2_debug.so) also checks the selection's lists
   and tags before the attention (indices in range and ascending, tags of the right class,
   counts equal to the budgets) and makes every stage call wait for its stream and return
   DA2_ERR_TIMEOUT at once when the error word is set. */
typedef struct da2_views {
  int N, bs, T, Tp, ny, nx, n8, n4, kv4;
  size_t tile8_qk, tile4_qk, tile8_v, tile4_v, sf_qk, sf_v;
  size_t q8, k8, v8, q4, k4, v4, sfq4, sfk4, sfv4;
  size_t sq, sk, sv, vamax, qavg, qmax, kavg, kmax;
  size_t tags, list8, list4, scores, err, total;
  int nm;               /* mixed KV blocks per query block */
  size_t listm;
  int n4max;            /* FP4 list length (n4 unless the adaptive budget is on) */
  size_t dlog;          /* draft logits scratch (N <= 1024), see below */
  int np;               /* its row length: N rounded up to a multiple of 4 */
  size_t qt, kt;        /* pooled Q / K split for the draft MMAs (N <= 1024), see below */
} da2_views;

/* Workspace bytes needed for `cfg` (host only, no CUDA call). */
da2_status da2_workspace_size(const da2_config* cfg, size_t* bytes);

/* Geometry and region offsets for `cfg` (host only, no CUDA call). */
da2_status da2_workspace_views(const da2_config* cfg, da2_views* views);

/* Operand preparation. q, k, v: device bf16 [B,H,T,d] ([B,T,H,d] with
   DA2_FLAG_LAYOUT_BTHD); ws: device workspace of at least
   da2_workspace_size bytes. Writes every operand, scale and pooled region of ws and
   clears its error word. Asynchronous on `stream`. */
da2_status da2_prepare(const da2_config* cfg, const void* q, const void* k, const void* v,
                       void* ws, size_t ws_bytes, cudaStream_t stream);

/* Draft maps and ranking on a prepared workspace: writes tags, list8, list4 (and scores
   with DA2_FLAG_EXPORT_SCORES). Asynchronous on `stream`. */
da2_status da2_draft_select(const da2_config* cfg, void* ws, size_t ws_bytes,
                            cudaStream_t stream);

/* Mixed-precision block-sparse attention on a prepared and selected workspace. out:
   device bf16 [B,H,T,d] ([B,T,H,d] with DA2_FLAG_LAYOUT_BTHD; every element is written). Bounded device waits that run out
   set the workspace error word (read it with da2_get_error). Asynchronous. */
da2_status da2_attention(const da2_config* cfg, void* ws, size_t ws_bytes, void* out,
                         cudaStream_t stream);

/* Debug aid (no counterpart in the paper): checks the output contract of
   da2_draft_select on a selected workspace before it reaches the attention. Per (b, h,
   query block) the FP8, mixed and FP4 lists must hold in-range, strictly ascending KV
   blocks tagged 2, 3 and 1, the FP4 list may end in -1 padding only after its last block,
   and the row must hold exactly n8 FP8 and nm mixed tags and n4..n4max FP4 tags. A
   violation sets bit 2 of the workspace error word (read it with da2_get_error). Reads
   only the workspace; asynchronous on `stream`. DA2_DEBUG builds run it inside
   da2_draft_select. */
da2_status da2_check_selection(const da2_config* cfg, void* ws, size_t ws_bytes,
                               cudaStream_t stream);

/* da2_prepare, da2_draft_select and da2_attention in order on one stream. */
da2_status da2_forward(const da2_config* cfg, const void* q, const void* k, const void* v,
                       void* out, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Host-buffer variant of da2_forward: copies q, k, v (host, bf16 [B,H,T,d]; pinned
   memory gives asynchronous copies) into the caller's device staging buffers dq, dk, dv,
   runs the three stages and copies the result from dout back to out_host. Heads being
   independent, it pipelines over up to 16 groups of heads: the copies in of one group and
   the copy out of another overlap the stages of a third (three internal streams, two
   sub-workspaces carved from ws, used alternately; each group's stages are exactly those
   of da2_forward on a configuration of its heads, so out_host is bit-identical to
   da2_forward's output). With fewer than 2 groups, or a workspace too small for two
   sub-workspaces, it runs everything on `stream`. Work queued on `stream` before the call
   runs first; the call synchronises `stream` before returning. Afterwards only the error
   word of ws (da2_get_error with cfg) is meaningful; the rest of ws holds the groups'
   layouts. ws_bytes must be at least da2_workspace_size(cfg). */
da2_status da2_forward_host(const da2_config* cfg, const void* q_host, const void* k_host,
                            const void* v_host, void* out_host, void* dq, void* dk,
                            void* dv, void* dout, void* ws, size_t ws_bytes,
                            cudaStream_t stream);

/* da2_forward without any device allocation, by the library or by the caller.
   No counterpart in the paper: this serves callers that cannot obtain device memory when
   they run the attention -- a plug-in inside a host framework that owns all device memory
   and exposes no allocator, or a serving loop that forbids cudaMalloc after start-up (it
   can synchronise the device and fail under fragmentation). The caller still passes q,
   k, v and out (device bf16 [B,H,T,d], 16-byte aligned); the workspace is a fixed 64 MiB
   device array inside the library, which every GPU that loads the library holds until
   the process exits. Configurations whose da2_workspace_size exceeds 64 MiB are rejected
   with DA2_ERR_SCRATCH_TOO_SMALL before anything is enqueued (the tiny workload and
   single-head 480p / 720p Wan-like layers fit; a full 40-head layer does not), and so is
   DA2_FLAG_EXPORT_SCORES (DA2_ERR_INVALID_ARG: the scores would stay in the hidden
   array). Every call looks up the array's device address on the current device
   (cudaGetSymbolAddress), so an address never outlives a device reset; the first call on
   a device also loads the library's device code there, so make it before any stream
   capture. Every call on a device shares the one array and leaves its contents behind;
   the path clears what must start at zero itself. Calls that overlap on the GPU
   (different streams, or several host threads on one device) race on the array and give
   wrong results: serialise them. Asynchronous on `stream` like da2_forward. Its device
   error word is read with da2_get_error(NULL, 0, cfg, stream, &word). */
da2_status da2_forward_noalloc(const da2_config* cfg, const void* q, const void* k,
                               const void* v, void* out, cudaStream_t stream);

/* Reads the workspace's device error word into *word and clears it (synchronises
   `stream`). Returns DA2_ERR_TIMEOUT if the word was non-zero. ws = NULL reads the word of
   the built-in array of da2_forward_noalloc (cfg as given to that call; ws_bytes is
   ignored). */
da2_status da2_get_error(void* ws, size_t ws_bytes, const da2_config* cfg,
                         cudaStream_t stream, uint32_t* word);

/* The cudaError_t of the calling host thread's most recent library call that returned
   DA2_ERR_CUDA (cudaSuccess if none). The library checks every launch with
   cudaGetLastError, which clears the runtime's own record, so this is where the code of,
   say, cudaErrorLaunchOutOfResources is kept. Host only, no CUDA call. */
int da2_last_cuda_error(void);

/* Static string naming a status. */
const char* da2_status_string(da2_status status);

#ifdef __cplusplus
}
#endif
#endif /* DA2_H */
