/*
 * FVAttn CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU statement of what the FVAttn
 * single-GPU hot path computes: video-aware block organisation, mean-pooled
 * block routing with Top-p plus a Top-k floor, masked attention over the
 * kept blocks, and the inverse reorder.  It exists so that tests, the smoke
 * check and the benchmark's CPU-baseline leg can check and time the CUDA
 * path.  Nothing in the product path may call it, and it shares no code,
 * header, table or constant with the CUDA sources.
 *
 * Sources (web pages about arXiv 2607.16190, "FVAttn: Adaptive Sparse
 * Attention with Runtime Load Balancing for Video Generation"):
 *   - paperlayer.ai summary, section 3 "FVAttn Design", item
 *     "Sparse-routing frontend": block reordering that keeps spatially
 *     adjacent tokens in nearby blocks, Top-p CDF thresholding, a Top-k floor.
 *   - paperlayer.ai summary, section 2 "Background and Related Work": Top-p
 *     keeps the smallest set of key blocks whose cumulative importance
 *     reaches p; the Top-k floor keeps a minimum budget; dynamic masks come
 *     from the current attention features.
 *   - paperlayer.ai summary, section 3, item "Pipeline": mask construction,
 *     then block-sparse attention, then restoration of the original layout.
 * Where the pages leave a step open, the readings taken are listed beside
 * the function that takes them.
 *
 * Arithmetic: fp64 throughout.  bf16 inputs are widened exactly to double.
 * Parallelism: OpenMP over independent rows / items only; every per-row or
 * per-item computation is sequential in the order written.
 *
 * Pins: every function here is checked by the CPU test-suite against
 * closed forms, brute force and library routines (numpy / torch fp64).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Geometry                                                            */
/* ------------------------------------------------------------------ */

typedef struct {
    int B, H, D, F, Hs, Ws, tf, th, tw; /* given */
    int Fp, Hp, Wp;                      /* padded video extents */
    int nbf, nby, nbx;                   /* tiles along frame, row, col */
    int bs, nb;                          /* tokens per block, blocks */
    long N, Npad;                        /* raster tokens, padded tokens */
    int order;                           /* 0: raster tile order, 1: Hilbert */
    int *tile_of_block;                  /* order 1: raster tile index of block b */
    int *block_of_tile;                  /* order 1: block index of raster tile t */
} og_geom;

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

static void og_make(og_geom *g, int B, int H, int D, int F, int Hs, int Ws,
                    int tf, int th, int tw) {
    g->B = B; g->H = H; g->D = D; g->F = F; g->Hs = Hs; g->Ws = Ws;
    g->tf = tf; g->th = th; g->tw = tw;
    g->nbf = ceil_div(F, tf);
    g->nby = ceil_div(Hs, th);
    g->nbx = ceil_div(Ws, tw);
    g->Fp = g->nbf * tf;
    g->Hp = g->nby * th;
    g->Wp = g->nbx * tw;
    g->bs = tf * th * tw;
    g->nb = g->nbf * g->nby * g->nbx;
    g->N = (long)F * Hs * Ws;
    g->Npad = (long)g->nb * g->bs;
    g->order = 0;
    g->tile_of_block = NULL;
    g->block_of_tile = NULL;
}

/* Index of cell (c[0], c[1], c[2]) along the 3-D Hilbert curve that fills a
 * cube of side 2^bits, after J. Skilling, "Programming the Hilbert curve"
 * (AIP Conf. Proc. 707, 2004): the coordinates are turned into the curve's
 * "transposed" index (an inverse-undo sweep from the top bit down, then Gray
 * encoding), whose bits, read top bit first and coordinate 0 first within a
 * bit, are the index. */
static unsigned long long og_hilbert3(const unsigned c_in[3], int bits) {
    unsigned c[3] = {c_in[0], c_in[1], c_in[2]};
    const unsigned top = 1u << (bits - 1);
    for (unsigned q = top; q > 1u; q >>= 1) {
        const unsigned low = q - 1u;
        for (int i = 0; i < 3; ++i) {
            if (c[i] & q) {
                c[0] ^= low;                       /* invert the low bits */
            } else {
                const unsigned t = (c[0] ^ c[i]) & low;   /* exchange low bits with c[0] */
                c[0] ^= t;
                c[i] ^= t;
            }
        }
    }
    for (int i = 1; i < 3; ++i) c[i] ^= c[i - 1];   /* Gray encode */
    unsigned t = 0;
    for (unsigned q = top; q > 1u; q >>= 1)
        if (c[2] & q) t ^= q - 1u;
    for (int i = 0; i < 3; ++i) c[i] ^= t;
    unsigned long long h = 0;
    for (int b = bits - 1; b >= 0; --b)
        for (int i = 0; i < 3; ++i) h = (h << 1) | ((c[i] >> b) & 1u);
    return h;
}

typedef struct { unsigned long long key; int tile; } og_hkey;

static int og_cmp_hkey(const void *pa, const void *pb) {
    const og_hkey *a = (const og_hkey *)pa, *b = (const og_hkey *)pb;
    return (a->key > b->key) - (a->key < b->key);
}

/* Hilbert block order (paperlayer.ai summary, section 3, "Sparse-routing
 * frontend": Hilbert-curve block reordering keeps spatially adjacent tokens
 * in nearby blocks).  Reading taken: the tile grid (frame, row, col) =
 * (nbf, nby, nbx) sits in the smallest cube of side 2^bits that holds it,
 * and blocks are numbered by increasing curve index of their tile.  Tokens
 * inside a tile keep raster order. */
static void og_block_order(int nbf, int nby, int nbx, int *tile_of_block, int *block_of_tile) {
    const int nb = nbf * nby * nbx;
    int side = nbf > nby ? nbf : nby;
    if (nbx > side) side = nbx;
    int bits = 1;
    while ((1 << bits) < side) ++bits;
    og_hkey *k = (og_hkey *)malloc(sizeof(og_hkey) * (size_t)nb);
    for (int t = 0; t < nb; ++t) {
        const unsigned c[3] = {(unsigned)(t / (nby * nbx)), (unsigned)((t / nbx) % nby), (unsigned)(t % nbx)};
        k[t].key = og_hilbert3(c, bits);
        k[t].tile = t;
    }
    qsort(k, (size_t)nb, sizeof(og_hkey), og_cmp_hkey);
    for (int b = 0; b < nb; ++b) {
        tile_of_block[b] = k[b].tile;
        if (block_of_tile) block_of_tile[k[b].tile] = b;
    }
    free(k);
}

static void og_set_order(og_geom *g, int order) {
    g->order = order;
    if (order == 1) {
        g->tile_of_block = (int *)malloc(sizeof(int) * (size_t)g->nb);
        g->block_of_tile = (int *)malloc(sizeof(int) * (size_t)g->nb);
        og_block_order(g->nbf, g->nby, g->nbx, g->tile_of_block, g->block_of_tile);
    }
}

static void og_free(og_geom *g) {
    free(g->tile_of_block);
    free(g->block_of_tile);
    g->tile_of_block = g->block_of_tile = NULL;
}

/* Exported: the Hilbert block order of a tile grid, tile_of_block[nb]. */
void oracle_block_order(int nbf, int nby, int nbx, int *tile_of_block) {
    og_block_order(nbf, nby, nbx, tile_of_block, NULL);
}

/* Video-aware block organisation (paperlayer.ai summary, section 3,
 * "Sparse-routing frontend").  Reading taken: the video is cut into
 * tf x th x tw spatio-temporal tiles; tiles are numbered in raster order
 * (tile-frame, tile-row, tile-col) and the tokens inside a tile in raster
 * order (frame, row, col).  Token (f, y, x) lands at position
 * block * bs + offset. */
static long og_tiled_pos(const og_geom *g, int f, int y, int x) {
    long block = ((long)(f / g->tf) * g->nby + (y / g->th)) * g->nbx + (x / g->tw);
    if (g->order == 1) block = g->block_of_tile[block];
    long offset = ((long)(f % g->tf) * g->th + (y % g->th)) * g->tw + (x % g->tw);
    return block * g->bs + offset;
}

/* The inverse question: which (f, y, x) sits at tiled position pos, and is
 * it a real token (1) or padding (0)? */
static int og_token_at(const og_geom *g, long pos, int *f, int *y, int *x) {
    long block = pos / g->bs;
    long offset = pos % g->bs;
    if (g->order == 1) block = g->tile_of_block[block];   /* the block's raster tile */
    int bx = (int)(block % g->nbx);
    int by = (int)((block / g->nbx) % g->nby);
    int bf = (int)(block / ((long)g->nbx * g->nby));
    int ox = (int)(offset % g->tw);
    int oy = (int)((offset / g->tw) % g->th);
    int of = (int)(offset / ((long)g->tw * g->th));
    *f = bf * g->tf + of;
    *y = by * g->th + oy;
    *x = bx * g->tw + ox;
    return (*f < g->F) && (*y < g->Hs) && (*x < g->Ws);
}

static double bf16_to_double(uint16_t u) {
    uint32_t bits = (uint32_t)u << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Number of real tokens in block `block`. */
static int og_block_valid(const og_geom *g, long block) {
    int n = 0, f, y, x;
    for (int o = 0; o < g->bs; ++o)
        n += og_token_at(g, block * g->bs + o, &f, &y, &x);
    return n;
}

/* Exported: derived geometry, as ints: Fp Hp Wp nbf nby nbx bs nb N Npad */
void oracle_geometry(int B, int H, int D, int F, int Hs, int Ws, int tf, int th, int tw,
                     long *out10) {
    og_geom g;
    og_make(&g, B, H, D, F, Hs, Ws, tf, th, tw);
    out10[0] = g.Fp; out10[1] = g.Hp; out10[2] = g.Wp;
    out10[3] = g.nbf; out10[4] = g.nby; out10[5] = g.nbx;
    out10[6] = g.bs; out10[7] = g.nb; out10[8] = g.N; out10[9] = g.Npad;
}

/* Exported: valid-token count of every block, int32[nb]. */
void oracle_block_valid_counts(int F, int Hs, int Ws, int tf, int th, int tw, int order, int *out) {
    og_geom g;
    og_make(&g, 1, 1, 1, F, Hs, Ws, tf, th, tw);
    og_set_order(&g, order);
    for (long b = 0; b < g.nb; ++b) out[b] = og_block_valid(&g, b);
    og_free(&g);
}

/* ------------------------------------------------------------------ */
/* Reorder / inverse reorder (bit copies of 16-bit elements)           */
/* ------------------------------------------------------------------ */

/* x: raster [B, N, H, D]  ->  out: tiled [B, H, Npad, D]; padding is zero. */
void oracle_reorder(const uint16_t *x, uint16_t *out,
                    int B, int H, int D, int F, int Hs, int Ws, int tf, int th, int tw, int order) {
    og_geom g;
    og_make(&g, B, H, D, F, Hs, Ws, tf, th, tw);
    og_set_order(&g, order);
    memset(out, 0, sizeof(uint16_t) * (size_t)B * H * g.Npad * D);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int f = 0; f < F; ++f)
            for (int y = 0; y < Hs; ++y)
                for (int xx = 0; xx < Ws; ++xx) {
                    long n = ((long)f * Hs + y) * Ws + xx;
                    long pos = og_tiled_pos(&g, f, y, xx);
                    for (int h = 0; h < H; ++h) {
                        const uint16_t *src = x + (((long)b * g.N + n) * H + h) * D;
                        uint16_t *dst = out + (((long)b * H + h) * g.Npad + pos) * D;
                        memcpy(dst, src, sizeof(uint16_t) * D);
                    }
                }
    og_free(&g);
}

/* t: tiled [B, H, Npad, D]  ->  x: raster [B, N, H, D]; padding is dropped. */
void oracle_inverse_reorder(const uint16_t *t, uint16_t *x,
                            int B, int H, int D, int F, int Hs, int Ws, int tf, int th, int tw, int order) {
    og_geom g;
    og_make(&g, B, H, D, F, Hs, Ws, tf, th, tw);
    og_set_order(&g, order);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int f = 0; f < F; ++f)
            for (int y = 0; y < Hs; ++y)
                for (int xx = 0; xx < Ws; ++xx) {
                    long n = ((long)f * Hs + y) * Ws + xx;
                    long pos = og_tiled_pos(&g, f, y, xx);
                    for (int h = 0; h < H; ++h) {
                        const uint16_t *src = t + (((long)b * H + h) * g.Npad + pos) * D;
                        uint16_t *dst = x + (((long)b * g.N + n) * H + h) * D;
                        memcpy(dst, src, sizeof(uint16_t) * D);
                    }
                }
    og_free(&g);
}

/* ------------------------------------------------------------------ */
/* Routing                                                             */
/* ------------------------------------------------------------------ */

/* Block mean-pooling of a tiled bf16 tensor (reading taken: the block
 * importance proxy is the mean of the block's real tokens; padding is
 * excluded from the mean).  t: tiled [B, H, Npad, D] bf16 bits;
 * out: [B, H, nb, D] double. */
void oracle_pool(const uint16_t *t, double *out,
                 int B, int H, int D, int F, int Hs, int Ws, int tf, int th, int tw, int order) {
    og_geom g;
    og_make(&g, B, H, D, F, Hs, Ws, tf, th, tw);
    og_set_order(&g, order);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < B * H; ++bh)
        for (int blk = 0; blk < g.nb; ++blk) {
            double *acc = out + ((long)bh * g.nb + blk) * D;
            for (int d = 0; d < D; ++d) acc[d] = 0.0;
            int n_valid = 0, f, y, x;
            for (int o = 0; o < g.bs; ++o) {
                long pos = (long)blk * g.bs + o;
                if (!og_token_at(&g, pos, &f, &y, &x)) continue;
                ++n_valid;
                const uint16_t *row = t + ((long)bh * g.Npad + pos) * D;
                for (int d = 0; d < D; ++d) acc[d] += bf16_to_double(row[d]);
            }
            for (int d = 0; d < D; ++d) acc[d] /= (double)n_valid;
        }
    og_free(&g);
}

/* Block scores: L[i][j] = scale * <qp_i, kp_j> per (b, h).  qp, kp: [BH, nb, D]
 * double; out: [BH, nb, nb] double. */
void oracle_logits(const double *qp, const double *kp, double *out,
                   int BH, int nb, int D, double scale) {
    #pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < BH; ++bh)
        for (int i = 0; i < nb; ++i) {
            const double *a = qp + ((long)bh * nb + i) * D;
            for (int j = 0; j < nb; ++j) {
                const double *b = kp + ((long)bh * nb + j) * D;
                double s = 0.0;
                for (int d = 0; d < D; ++d) s += a[d] * b[d];
                out[((long)bh * nb + i) * nb + j] = s * scale;
            }
        }
}

typedef struct { float key; int idx; } og_entry;

/* Order pi: larger logit first; equal fp32 logits go to the lower block
 * index first.  The order is on the fp32 logits themselves, not on the
 * probabilities, because rounding exp() could merge distinct logits. */
static int og_cmp(const void *pa, const void *pb) {
    const og_entry *a = (const og_entry *)pa, *b = (const og_entry *)pb;
    if (a->key > b->key) return -1;
    if (a->key < b->key) return 1;
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

static int og_cmp_int(const void *pa, const void *pb) {
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

/* Top-p with a Top-k floor on one row of fp32 logits (paperlayer.ai summary,
 * section 2: Top-p keeps the smallest cumulative-importance set, the Top-k
 * safety floor keeps a minimum budget; section 3: Top-p CDF thresholding).
 *   P_j   = exp(L_j - max L) / sum_i exp(L_i - max L)          (double)
 *   c_r   = P_pi(1) + ... + P_pi(r), summed left to right       (double)
 *   m_p   = min { r : c_r >= p }   ("reaches p": inclusive)
 *           p >= 1 gives m_p = nb (floating sums may never reach 1)
 *           p <= 0 gives m_p = 0: Top-p off, the fixed Top-k mode
 *   m     = max(m_p, min(k, nb))  (the union of two prefixes of pi is the
 *                                  longer prefix)
 *   m    <- min(nb, m + k_extra)  (importance-order augmentation: the next
 *                                  k_extra blocks of pi, this build's
 *                                  single-GPU reading of the pages' slack
 *                                  augmentation; k_extra = 0 leaves m)
 *   kept  = first m of pi, written out in ascending block index
 * Near-tie flag: set when c_{m_p} or c_{m_p - 1} is within `tie_band` of p.
 * Returns m; writes m_p and the flag. */
static int og_select_row(const float *L, int nb, double p, int k, int k_extra, double tie_band,
                         int *idx_out, int *mp_out, int *tie_out, og_entry *e, double *prob) {
    for (int j = 0; j < nb; ++j) { e[j].key = L[j]; e[j].idx = j; }
    qsort(e, (size_t)nb, sizeof(og_entry), og_cmp);
    double lmax = (double)e[0].key;
    double z = 0.0;
    for (int r = 0; r < nb; ++r) { prob[r] = exp((double)e[r].key - lmax); z += prob[r]; }
    for (int r = 0; r < nb; ++r) prob[r] /= z;
    int mp = nb, tie = 0;
    if (p <= 0.0) {
        mp = 0;
    } else if (p < 1.0) {
        double c = 0.0, c_prev = 0.0;
        mp = nb;
        for (int r = 0; r < nb; ++r) {
            c_prev = c;
            c += prob[r];
            if (c >= p) { mp = r + 1; break; }
        }
        double c_mp = c;
        if (fabs(c_mp - p) <= tie_band) tie = 1;
        if (mp > 1 && fabs(c_prev - p) <= tie_band) tie = 1;
    }
    int kf = k < nb ? k : nb;
    int m = mp > kf ? mp : kf;
    m = (k_extra > nb - m) ? nb : m + k_extra;
    for (int r = 0; r < m; ++r) idx_out[r] = e[r].idx;
    qsort(idx_out, (size_t)m, sizeof(int), og_cmp_int);
    *mp_out = mp;
    *tie_out = tie;
    return m;
}

/* Exported: select on `rows` rows of fp32 logits [rows, nb].
 * idx: [rows, nb] (first cnt entries written, rest set to -1);
 * cnt, mp, tie: [rows]. */
void oracle_select_aug(const float *L, int rows, int nb, double p, int k, int k_extra, double tie_band,
                       int *idx, int *cnt, int *mp, int *tie) {
    #pragma omp parallel
    {
        og_entry *e = (og_entry *)malloc(sizeof(og_entry) * (size_t)nb);
        double *prob = (double *)malloc(sizeof(double) * (size_t)nb);
        #pragma omp for schedule(static)
        for (int r = 0; r < rows; ++r) {
            int *row_idx = idx + (long)r * nb;
            for (int j = 0; j < nb; ++j) row_idx[j] = -1;
            cnt[r] = og_select_row(L + (long)r * nb, nb, p, k, k_extra, tie_band, row_idx,
                                   &mp[r], &tie[r], e, prob);
        }
        free(e);
        free(prob);
    }
}

/* Exported: Top-p with the Top-k floor only (k_extra = 0). */
void oracle_select(const float *L, int rows, int nb, double p, int k, double tie_band,
                   int *idx, int *cnt, int *mp, int *tie) {
    oracle_select_aug(L, rows, nb, p, k, 0, tie_band, idx, cnt, mp, tie);
}

/* ------------------------------------------------------------------ */
/* Attention                                                           */
/* ------------------------------------------------------------------ */

/* Masked attention for selected items (paperlayer.ai summary, section 2:
 * dynamic block-sparse attention; section 3 "Pipeline": block-sparse
 * attention runs on the materialised mask).  Item = (b, h, query block i),
 * flattened as (b*H + h)*nb + i.  For every real query token t of block i:
 *   o_t = sum_{u in U_i} softmax_u(scale * q_t . k_u) v_u,
 * where U_i holds the real tokens of the kept key blocks of row i.  Padding
 * query rows are written as zero.  qt, kt, vt: tiled [B, H, Npad, D] bf16
 * bits; kv_idx: [B*H*nb, nb]; kv_cnt: [B*H*nb]; out: [n_items, bs, D]. */
void oracle_attention(const uint16_t *qt, const uint16_t *kt, const uint16_t *vt,
                      const int *kv_idx, const int *kv_cnt, const long *items, int n_items,
                      double scale, double *out,
                      int B, int H, int D, int F, int Hs, int Ws, int tf, int th, int tw, int order) {
    og_geom g;
    og_make(&g, B, H, D, F, Hs, Ws, tf, th, tw);
    og_set_order(&g, order);
    const int bs = g.bs;
    #pragma omp parallel
    {
        long max_keys = g.Npad;
        double *s = (double *)malloc(sizeof(double) * (size_t)max_keys);
        long *key_pos = (long *)malloc(sizeof(long) * (size_t)max_keys);
        double *qrow = (double *)malloc(sizeof(double) * (size_t)D);
        #pragma omp for schedule(dynamic, 1) collapse(2)
        for (int it = 0; it < n_items; ++it)
            for (int o = 0; o < bs; ++o) {
                long item = items[it];
                long bh = item / g.nb;
                int i = (int)(item % g.nb);
                double *orow = out + ((long)it * bs + o) * D;
                int f, y, x;
                if (!og_token_at(&g, (long)i * bs + o, &f, &y, &x)) {
                    for (int d = 0; d < D; ++d) orow[d] = 0.0;
                    continue;
                }
                const uint16_t *q = qt + (bh * g.Npad + (long)i * bs + o) * D;
                for (int d = 0; d < D; ++d) qrow[d] = bf16_to_double(q[d]);
                /* gather the real key tokens of the kept blocks */
                long nk = 0;
                int c = kv_cnt[item];
                const int *list = kv_idx + item * g.nb;
                for (int r = 0; r < c; ++r) {
                    int j = list[r];
                    for (int u = 0; u < bs; ++u) {
                        long pos = (long)j * bs + u;
                        if (og_token_at(&g, pos, &f, &y, &x)) key_pos[nk++] = pos;
                    }
                }
                double smax = -INFINITY;
                for (long u = 0; u < nk; ++u) {
                    const uint16_t *kr = kt + (bh * g.Npad + key_pos[u]) * D;
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += qrow[d] * bf16_to_double(kr[d]);
                    s[u] = acc * scale;
                    if (s[u] > smax) smax = s[u];
                }
                double z = 0.0;
                for (long u = 0; u < nk; ++u) { s[u] = exp(s[u] - smax); z += s[u]; }
                for (int d = 0; d < D; ++d) orow[d] = 0.0;
                for (long u = 0; u < nk; ++u) {
                    const uint16_t *vr = vt + (bh * g.Npad + key_pos[u]) * D;
                    double w = s[u] / z;
                    for (int d = 0; d < D; ++d) orow[d] += w * bf16_to_double(vr[d]);
                }
            }
        free(s);
        free(key_pos);
        free(qrow);
    }
    og_free(&g);
}

/* Exported: number of OpenMP threads the oracle will use. */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
