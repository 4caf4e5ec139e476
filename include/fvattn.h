/*
 * fvattn.h -- C ABI of the FVAttn single-GPU hot path on B200 (sm_100a).
 *
 * FVAttn ("FVAttn: Adaptive Sparse Attention with Runtime Load Balancing
 * for Video Generation", arXiv 2607.16190) builds, per attention layer, a
 * video-aware block organisation, a Top-p plus Top-k-floor block mask from
 * the current attention features, and then runs block-sparse attention on
 * that mask (paperlayer.ai summary, section 3 "FVAttn Design", items
 * "Pipeline" and "Sparse-routing frontend"; section 2 "Background and
 * Related Work", items on Top-p, Top-k and dynamic block-sparse attention).
 * This library exposes the four single-GPU steps of that path:
 *
 *   fvattn_reorder          raster tokens -> spatio-temporal tiles
 *   fvattn_route            block mean-pooling, block scores, Top-p + Top-k
 *   fvattn_sparse_attn      block-sparse flash attention on the kept blocks
 *   fvattn_inverse_reorder  tiles -> raster tokens
 *
 * and fused forms of the first two and last two steps
 * (fvattn_reorder_route: reorder of Q and K and routing in one pass over
 * them; fvattn_sparse_attn_raster: attention writing raster rows), with the
 * same results bit for bit.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers, 16-byte aligned, contiguous.
 *     bf16 tensors are passed as void* holding IEEE bfloat16 values.
 *   - The caller owns (allocates and frees) every buffer, including the
 *     workspaces.  The library allocates and frees no device memory.
 *   - Every call is asynchronous on the given stream (a cudaStream_t; NULL
 *     is the legacy default stream) and never synchronises it, except
 *     fvattn_get_status.
 *   - Return value: FVATTN_OK or an error code below.  Argument errors are
 *     detected on the host before anything is launched.  Errors raised
 *     inside a kernel (a bounded wait that ran out, a kv index out of range)
 *     are recorded in a device status word read by fvattn_get_status.
 *   - Nothing here falls back to the CPU.
 *
 * Geometry (notation of the pages' video DiT setting): a layer has B
 * sequences, H heads of dimension D, and a latent video of F frames of
 * Hs x Ws tokens, in raster (frame, row, col) order: N = F*Hs*Ws tokens.
 * Tiles are tf x th x tw tokens; the video is zero-padded up to
 * Fp = ceil(F/tf)*tf (likewise Hp, Wp).  A block is one tile of
 * bs = tf*th*tw tokens; tiles are numbered in raster tile order and the
 * tokens inside a tile in raster order.  nb = Npad/bs blocks per head;
 * every block holds at least one real token.
 */
#ifndef FVATTN_H
#define FVATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque stream handle: pass a cudaStream_t. */
typedef struct CUstream_st *fvattn_stream_t;

enum {
    FVATTN_OK = 0,
    FVATTN_ERR_INVALID = 1,     /* null / misaligned pointer, bad p or k, workspace too small */
    FVATTN_ERR_UNSUPPORTED = 2, /* geometry outside the supported range */
    FVATTN_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed */
    FVATTN_ERR_TIMEOUT = 4,     /* a bounded device wait ran out (kernel returned early) */
    FVATTN_ERR_BOUNDS = 5       /* a kv_idx / kv_cnt entry was out of range */
};

typedef struct {
    /* set by the caller */
    int B, H, D;          /* batch, heads, head dim (64 or 128) */
    int F, Hs, Ws;        /* latent frames, rows, cols */
    int tf, th, tw;       /* tile extent; bs = tf*th*tw in {16, 32, 64, 128} */
    /* filled by fvattn_geom_init */
    int Fp, Hp, Wp;       /* padded extents */
    int nbf, nby, nbx;    /* tiles along frame, row, col */
    int bs, nb;           /* tokens per block, blocks per head (nb <= 2560) */
    long long N, Npad;    /* raster tokens, padded tokens (= nb*bs) */
    /* optional, set by the caller after fvattn_geom_init: device table of
     * 2*nb int32 written by fvattn_block_order; NULL numbers the tiles in
     * raster tile order (fvattn_geom_init sets NULL) */
    const int32_t *order;
} fvattn_geom;

/* Validate the caller-set fields and fill the derived ones.
 * Returns FVATTN_ERR_INVALID for non-positive sizes, FVATTN_ERR_UNSUPPORTED
 * for D not in {64, 128}, bs not in {16, 32, 64, 128} or nb > 2560. */
int fvattn_geom_init(fvattn_geom *g);

/* Hilbert block order (paperlayer.ai summary, section 3, "Sparse-routing
 * frontend": Hilbert-curve block reordering places spatially adjacent tokens
 * in nearby blocks).  Writes into `table` (device, 2*nb int32, 16-byte
 * aligned): [0, nb) the raster tile index ((f/tf)*nby + y/th)*nbx + x/tw of
 * each block, [nb, 2nb) the block of each raster tile.  Blocks are numbered
 * by increasing index of their tile along the 3-D Hilbert curve of the
 * smallest cube of side 2^b holding the (nbf, nby, nbx) tile grid.  Set
 * g->order = table afterwards to use it in every call; tokens inside a tile
 * keep raster order.  Asynchronous on `stream`. */
int fvattn_block_order(const fvattn_geom *g, int32_t *table, fvattn_stream_t stream);

/* Video-aware block organisation (paperlayer.ai summary, section 3,
 * "Sparse-routing frontend": spatially adjacent tokens share a block).
 *   x       [B, N, H, D] bf16, raster token order (the DiT's layout)
 *   x_tiled [B, H, Npad, D] bf16; token (f, y, x) of head h goes to row
 *           block*bs + offset, block = ((f/tf)*nby + y/th)*nbx + x/tw
 *           (or that tile's block in g->order when set),
 *           offset = ((f%tf)*th + y%th)*tw + x%tw; padding rows are zero.
 * Bit copy.  x and x_tiled must not overlap. */
int fvattn_reorder(const fvattn_geom *g, const void *x, void *x_tiled, fvattn_stream_t stream);

/* Restoration of the original layout (paperlayer.ai summary, section 3,
 * "Pipeline", last step): the exact inverse of fvattn_reorder on real
 * tokens; padding rows are dropped.
 *   o_tiled [B, H, Npad, D] bf16  ->  o [B, N, H, D] bf16.  Bit copy. */
int fvattn_inverse_reorder(const fvattn_geom *g, const void *o_tiled, void *o,
                           fvattn_stream_t stream);

/* Bytes of device workspace fvattn_route needs: the pooled Q and K split
 * into tf32 high and low parts (4 x [B, H, nb, D] fp32) and the logits
 * ([B, H, nb, nb] fp32). */
size_t fvattn_route_workspace_size(const fvattn_geom *g);

/* Sparse-routing frontend (paperlayer.ai summary, section 3,
 * "Sparse-routing frontend": Top-p CDF thresholding and a Top-k floor;
 * section 2: Top-p keeps the smallest cumulative-importance set, the Top-k
 * safety floor a minimum budget).  Per (b, h):
 *   Qp[i] = mean of the real tokens of query block i (fp32), Kp likewise;
 *   L[i][j] = scale * Qp[i] . Kp[j]                      (fp32; on the tensor
 *             cores as three tf32 products hi*hi + hi*lo + lo*hi of the
 *             split Qp = hi + lo, Kp likewise: about fp32 accuracy)
 *   order blocks of row i by L descending, equal L by lower j;
 *   P = softmax(L[i]); m_p = smallest prefix whose mass reaches p
 *   (m_p = nb when p >= 1); m = max(m_p, min(k_floor, nb));
 *   kv_idx[b,h,i,0..m) = the first m blocks of that order, ascending;
 *   kv_cnt[b,h,i] = m.
 * Arguments:
 *   q_tiled, k_tiled  [B, H, Npad, D] bf16 from fvattn_reorder
 *   p                 in (0, 1]
 *   k_floor           >= 1
 *   scale             softmax scale (normally 1/sqrt(D)); must be finite
 *   kv_idx            [B, H, nb, nb] int32; entries at and after kv_cnt are
 *                     left unwritten
 *   kv_cnt            [B, H, nb] int32
 *   q_pool, k_pool    optional [B, H, nb, D] fp32 outputs (may be NULL)
 *   logits            optional [B, H, nb, nb] fp32 output of L (may be NULL)
 *   workspace         device scratch of >= fvattn_route_workspace_size bytes,
 *                     256-byte aligned (always required)
 * Logits must be finite (NaN inputs give an unspecified mask). */
int fvattn_route(const fvattn_geom *g, const void *q_tiled, const void *k_tiled,
                 double p, int k_floor, float scale,
                 int32_t *kv_idx, int32_t *kv_cnt,
                 float *q_pool, float *k_pool, float *logits,
                 void *workspace, size_t ws_bytes, fvattn_stream_t stream);

/* Routing variants, this build's single-GPU readings of two passages
 * (paperlayer.ai summary, section 2, "Sparse Attention": Top-k keeps a fixed
 * number of blocks, against which Top-p is compared; section 3, "Slack-Aware
 * Sparse Augmentation": extra high-value blocks taken in routing's
 * importance order):
 *   p = 0        fixed Top-k mode: m_p = 0, so m = min(k_floor, nb);
 *   k_extra >= 0 importance-order augmentation: the next k_extra blocks of
 *                the same order are kept too, m = min(nb, m + k_extra).
 * p in [0, 1], k_floor >= 1, k_extra >= 0; otherwise as fvattn_route
 * (fvattn_route is this call with k_extra = 0 and p > 0). */
int fvattn_route_aug(const fvattn_geom *g, const void *q_tiled, const void *k_tiled,
                     double p, int k_floor, int k_extra, float scale,
                     int32_t *kv_idx, int32_t *kv_cnt,
                     float *q_pool, float *k_pool, float *logits,
                     void *workspace, size_t ws_bytes, fvattn_stream_t stream);

/* Reorder of Q and K fused with routing (paperlayer.ai summary, section 3,
 * "Pipeline": the video-aware reorder comes first and the sparse-routing
 * frontend pools the reordered blocks; here both happen in one pass over
 * the raster tensors, which are read once).
 *   q, k              raster [B, N, H, D] bf16 device tensors (as for
 *                     fvattn_reorder), 16-byte aligned, read only
 *   q_tiled, k_tiled  tiled [B, H, Npad, D] bf16 outputs, two distinct
 *                     buffers: bit for bit what fvattn_reorder writes
 *   the rest          as fvattn_route_aug.
 * The pooled means are bit-identical to pooling the tiles afterwards, so
 * kv_idx / kv_cnt equal those of fvattn_reorder x 2 + fvattn_route_aug on
 * the same inputs.  Launches fvattn_route_kernel_launches kernels.  Null or
 * misaligned pointers, q_tiled == k_tiled, and the parameter errors of
 * fvattn_route_aug return FVATTN_ERR_INVALID before any launch. */
int fvattn_reorder_route(const fvattn_geom *g, const void *q, const void *k, void *q_tiled, void *k_tiled,
                         double p, int k_floor, int k_extra, float scale,
                         int32_t *kv_idx, int32_t *kv_cnt,
                         float *q_pool, float *k_pool, float *logits,
                         void *workspace, size_t ws_bytes, fvattn_stream_t stream);

/* Host <-> device copy of a head slice of a raster tensor, for pipelining a
 * layer by head groups (plumbing; no part of the method).  Heads
 * [h0, h0 + nh) of a raster [B, N, H, D] bf16 tensor in host memory (page
 * locked for asynchrony) go to / come from a device [B, N, nh, D] bf16
 * buffer; g gives B, N, H, D of the full tensor.  to_device = 1: src is the
 * host tensor, dst the device slice; 0: src is the device slice, dst the
 * host tensor.  One 2-D asynchronous copy on `stream`. */
int fvattn_copy_heads(const fvattn_geom *g, int h0, int nh, const void *src, void *dst, int to_device,
                      fvattn_stream_t stream);

/* Number of kernel launches one fvattn_route call makes for this geometry
 * (pooling, scoring, selection); 0 for a null pointer. */
int fvattn_route_kernel_launches(const fvattn_geom *g);

/* Bytes of device workspace fvattn_sparse_attn needs: the work list (item
 * order, head cost and order, counter), the blocks' real extents and, for
 * bs < 128, the union of each query group's kv lists (nb entries of 4 bytes
 * per group: 255 MB for the 40-head CFG layer at nb = 1260) and its size. */
size_t fvattn_attn_workspace_size(const fvattn_geom *g);

/* Number of CTAs (one per SM) the persistent attention kernel launches on
 * the current device; the length of each half of sm_stats. */
int fvattn_num_sms(void);

/* Dynamic block-sparse attention (paperlayer.ai summary, section 2,
 * "Sparse Attention": dynamic block-sparse attention; section 3,
 * "Pipeline": it runs on the materialised mask).  For each (b, h, query
 * block i) and each real or padding query row t of block i:
 *   O_t = softmax_u(scale * q_t . k_u) v_u  over the real tokens u of the
 *         kv_cnt[b,h,i] blocks kv_idx[b,h,i,0..cnt)
 * computed with bf16 tensor-core products, fp32 online softmax and fp32
 * accumulation, written as bf16.  scale must be finite and > 0.  Work items
 * are taken longest-first by a persistent kernel with one CTA per SM.  For
 * bs < 128 an item is a 128-row tile of 128 / bs consecutive query blocks
 * that walks the union of their kv lists, each row masked to its own
 * block's list (the order of a list does not matter).  The output bits
 * depend only on the inputs: not on which CTA takes an item, nor on how the
 * heads of a layer are split across calls.
 *   q_t, k_t, v_t  [B, H, Npad, D] bf16 from fvattn_reorder (padding zero)
 *   kv_idx, kv_cnt as written by fvattn_route (each row: cnt in [1, nb],
 *                  distinct indices in [0, nb)); out-of-range entries set
 *                  FVATTN_ERR_BOUNDS in the status word and are skipped
 *   o_t            [B, H, Npad, D] bf16 output (all rows written)
 *   sm_stats       optional (may be NULL) uint64[2 * fvattn_num_sms()]:
 *                  [0, n) busy nanoseconds of each CTA, [n, 2n) kv blocks
 *                  each CTA walked (for bs < 128: union blocks per tile)
 *   workspace      >= fvattn_attn_workspace_size bytes, 256-byte aligned */
int fvattn_sparse_attn(const fvattn_geom *g, const void *q_t, const void *k_t, const void *v_t,
                       const int32_t *kv_idx, const int32_t *kv_cnt, float scale,
                       void *o_t, unsigned long long *sm_stats,
                       void *workspace, size_t ws_bytes, fvattn_stream_t stream);

/* fvattn_sparse_attn with the inverse reorder fused into its epilogue
 * (paperlayer.ai summary, section 3, "Pipeline": attention, then
 * restoration of the original layout): each output row goes straight to its
 * raster position, and padding rows are not written.
 *   o  [B, N, H, D] bf16, the same bits fvattn_sparse_attn followed by
 *      fvattn_inverse_reorder would write.
 * Other arguments and errors as fvattn_sparse_attn.  It needs no tiled O
 * buffer (865 MB at the 720p layer); on B200 its scattered raster stores make
 * the attention step about 3% slower than fvattn_sparse_attn plus
 * fvattn_inverse_reorder. */
int fvattn_sparse_attn_raster(const fvattn_geom *g, const void *q_t, const void *k_t, const void *v_t,
                              const int32_t *kv_idx, const int32_t *kv_cnt, float scale,
                              void *o, unsigned long long *sm_stats,
                              void *workspace, size_t ws_bytes, fvattn_stream_t stream);

/* Maximum scratch, in bytes, of fvattn_sparse_attn_noalloc (2 MiB): enough
 * for fvattn_attn_workspace_size(g) of up to about 500 000 work items
 * (B*H*nb) at bs = 128 (e.g. B*H <= 200 at nb = 2560).  For bs < 128 the
 * query groups' union lists (B*H*ceil(nb*bs/128)*nb*4 bytes) count too: a
 * 40-head layer fits up to nb = 160 at bs = 64, 224 at bs = 32 and 318 at
 * bs = 16. */
#define FVATTN_NOALLOC_SCRATCH_BYTES (2u * 1024u * 1024u)

/* fvattn_sparse_attn without a workspace argument, for callers that cannot
 * allocate device memory (a plugin whose host framework owns all device
 * memory, a C caller with no device allocator, code that must not call
 * cudaMalloc once running).  The pages have no counterpart: this is a
 * packaging variant of the same computation and kernels.
 *   - Scratch: a device array of FVATTN_NOALLOC_SCRATCH_BYTES inside the
 *     library, held by every GPU that loads it until the process exits.  The
 *     call allocates nothing (no cudaMalloc, cudaFree or allocating library
 *     routine).
 *   - The first call on a device looks the array's device address up with
 *     cudaGetSymbolAddress (with that device current); make that first call
 *     before any stream capture.
 *   - Every call on a device shares the one array and fully rewrites what it
 *     reads, resetting its item counter to zero.  Calls that overlap on the
 *     GPU (different streams, or different host threads) race on it and must
 *     be serialised by the caller.
 *   - Returns FVATTN_ERR_UNSUPPORTED, before launching anything, when
 *     fvattn_attn_workspace_size(g) exceeds FVATTN_NOALLOC_SCRATCH_BYTES;
 *     otherwise the arguments and results are those of fvattn_sparse_attn. */
int fvattn_sparse_attn_noalloc(const fvattn_geom *g, const void *q_t, const void *k_t, const void *v_t,
                               const int32_t *kv_idx, const int32_t *kv_cnt, float scale,
                               void *o_t, unsigned long long *sm_stats, fvattn_stream_t stream);

/* Synchronise `stream`, read and clear the device status words (one per
 * library source file whose kernels record errors), and return the first
 * error found (FVATTN_OK, FVATTN_ERR_TIMEOUT or FVATTN_ERR_BOUNDS), or
 * FVATTN_ERR_CUDA if the synchronisation itself failed. */
int fvattn_get_status(fvattn_stream_t stream);

/* Fault injection for tests of the failure path (the pages have no
 * counterpart; it exists so that a test can make a device wait run out
 * without faulting, trapping or hanging the GPU).  Process-wide settings read
 * by every later fvattn_sparse_attn launch (and its raster and no-alloc
 * forms):
 *   wait_limit_ns  bound of every wait inside the attention kernel, in
 *                  nanoseconds; 0 restores the default (4 s)
 *   flags          0, or FVATTN_HOOK_SKIP_V_LOADS: the kernel's V-loading
 *                  warp leaves at once without loading or signalling
 *                  anything, so the wait of the PV issuer for V runs out.
 * A wait that runs out records FVATTN_ERR_TIMEOUT; every role of the CTA
 * then leaves its loop, waits for its own copies and MMAs in flight and
 * releases its tensor memory, and the kernel returns (its output is
 * unspecified).  Call fvattn_test_hook(0, 0) to return to normal operation.
 * Returns FVATTN_ERR_INVALID for unknown flags. */
#define FVATTN_HOOK_SKIP_V_LOADS 1
int fvattn_test_hook(unsigned long long wait_limit_ns, int flags);

/* Static string naming a status code. */
const char *fvattn_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* FVATTN_H */
