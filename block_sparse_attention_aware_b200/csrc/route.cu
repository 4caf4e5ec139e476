// Sparse-routing frontend of FVAttn (paperlayer.ai summary, section 3
// "FVAttn Design", item "Sparse-routing frontend": Top-p CDF thresholding of
// each query block's similarity distribution plus a Top-k floor; section 2:
// Top-p keeps the smallest cumulative-importance set, the Top-k safety floor
// a minimum budget; dynamic masks come from the current attention features).
//
// Three kernels:
//   pool_kernel    HBM-bound.  One warp per (tensor, b, h, block) sums the
//                  block's real rows with 16-byte loads, all issued before the
//                  first add (padding rows are never read), and writes the fp32
//                  mean split into its tf32 part and the exact remainder.
//   score_kernel   L = scale * Qp Kp^T per (b, h) on the tensor cores
//                  (tcgen05 kind::tf32, TMEM accumulators) as three tf32
//                  products hi*hi + hi*lo + lo*hi: about fp32 accuracy.
//   select_kernel  One warp per (b, h, query block) row, the row's logits and
//                  their masses e_j = exp(L_j - max L) in registers.  The
//                  weight of a set {L >= t} is an exact fixed-point integer (a
//                  lane's float partial sum scaled by 2^40, summed across the
//                  warp), so it is monotone in t and identical on every lane.
//                  The Top-p crossing (first prefix, logit descending then
//                  index ascending, whose mass reaches p * total) is bracketed
//                  by bisection on t with one warp reduction a step, until at
//                  most 32 entries remain, which the warp sorts (bitonic on
//                  64-bit order keys) and scans; the min(k, nb)-th entry (Top-k
//                  floor) is found the same way with counts when the Top-p
//                  prefix is shorter.  No shared-memory atomics.  The kept
//                  indices are written in ascending order with ballots.
//
// fvattn_reorder_route replaces the pooling kernel by reorder_pool_kernel,
// which reads raster Q and K once, writes their tiles and pools the same rows
// on the way (the reorder and pooling steps of the pages' pipeline in one
// pass).
#include <cstring>

#include "common.cuh"
#include "ptx.cuh"
#include "sync.cuh"
#include "tmap.cuh"

namespace fv {

// ------------------------------------------------------------------ pooling

// One warp per (tensor, b, h, block); 8 warps per CTA.  A lane owns one
// 16-byte column slice (D/8 slices per row) of every (32 / (D/8))-th row, so
// one warp instruction reads 512 contiguous bytes; full tiles issue all their
// loads before the first add.
struct PoolOut {
    float* hi[2];     // [q, k]: tf32 part of the mean (low 13 mantissa bits cleared)
    float* lo[2];     // [q, k]: mean - hi (exact)
    float* mean[2];   // [q, k]: the fp32 mean itself, or null
};

// Mean of a block's rows from the lanes' fp32 pair sums (lane l holds column
// slice l % (D/8) of every (32 / (D/8))-th row): reduce across the lanes of a
// slice, divide by the real-row count, write the tf32 part, the exact
// remainder and, if asked, the mean.
template <int D>
__device__ __forceinline__ void pool_write(const unsigned long long (&acc2)[4], int lane, int real_rows,
                                           long long dst_off, bool is_k, const PoolOut& out) {
    constexpr int VPR = D / 8;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) f2_unpack(acc2[e], acc[2 * e], acc[2 * e + 1]);
    // lanes with the same column slice hold partial sums of different rows
#pragma unroll
    for (int o = VPR; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (lane < VPR) {
        const float inv = 1.0f / static_cast<float>(real_rows);
        float m[8], h[8], l[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            m[e] = acc[e] * inv;
            h[e] = __uint_as_float(__float_as_uint(m[e]) & 0xffffe000u);
            l[e] = m[e] - h[e];
        }
        const long long o = dst_off + lane * 8;
        float* mp = is_k ? out.mean[1] : out.mean[0];
        float4* dh = reinterpret_cast<float4*>((is_k ? out.hi[1] : out.hi[0]) + o);
        float4* dl = reinterpret_cast<float4*>((is_k ? out.lo[1] : out.lo[0]) + o);
        dh[0] = make_float4(h[0], h[1], h[2], h[3]);
        dh[1] = make_float4(h[4], h[5], h[6], h[7]);
        dl[0] = make_float4(l[0], l[1], l[2], l[3]);
        dl[1] = make_float4(l[4], l[5], l[6], l[7]);
        if (mp) {
            float4* dm = reinterpret_cast<float4*>(mp + o);
            dm[0] = make_float4(m[0], m[1], m[2], m[3]);
            dm[1] = make_float4(m[4], m[5], m[6], m[7]);
        }
    }
}

// Adds the 8 bf16 of a 16-byte vector to the lane's fp32 pair sums.
__device__ __forceinline__ void pool_add(unsigned long long (&acc2)[4], const uint4& u) {
    const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        // a bf16 is the top half of the fp32 with the same value
        const float lo = __uint_as_float(wds[e] << 16), hi = __uint_as_float(wds[e] & 0xffff0000u);
        acc2[e] = f2_add(acc2[e], f2_pack(lo, hi));
    }
}

template <int D>
__global__ void __launch_bounds__(256, 4) pool_kernel(Geo g, const __nv_bfloat16* __restrict__ qt,
                                                   const __nv_bfloat16* __restrict__ kt, PoolOut out) {
    constexpr int VPR = D / 8;             // 16-byte vectors per row
    constexpr int RPI = 32 / VPR;          // rows per warp instruction
    constexpr int UNR = 8;                 // loads in flight per lane
    pdl_launch_dependents();   // the score kernel may be scheduled as this grid drains
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long unit = static_cast<long long>(blockIdx.x) * 8 + warp;   // (tensor, bh, blk) flattened
    const long long per_tensor = static_cast<long long>(g.B) * g.H * g.nb;
    if (unit >= 2 * per_tensor) return;
    const bool is_k = unit >= per_tensor;
    const long long ub = is_k ? unit - per_tensor : unit;
    const long long bh = ub / g.nb;
    const int blk = static_cast<int>(ub - bh * g.nb);
    const uint4* src = reinterpret_cast<const uint4*>((is_k ? kt : qt) +
                                                      (bh * g.Npad + static_cast<long long>(blk) * g.bs) * D);
    const int vec = lane % VPR;
    const int r0 = lane / VPR;
    const int tile = tile_of_block(g, blk);
    const int bx = tile % g.nbx, by = (tile / g.nbx) % g.nby, bf = tile / (g.nbx * g.nby);
    const int nf = min(g.tf, g.F - bf * g.tf);
    const int ny = min(g.th, g.Hs - by * g.th);
    const int nx = min(g.tw, g.Ws - bx * g.tw);
    const bool full = nf == g.tf && ny == g.th && nx == g.tw;
    unsigned long long acc2[4];   // fp32 pairs (column 2e, 2e + 1) of this lane's slice
#pragma unroll
    for (int e = 0; e < 4; ++e) acc2[e] = 0ull;
    const int steps = g.bs / RPI;          // warp instructions per tile
    for (int s0 = 0; s0 < steps; s0 += UNR) {
        uint4 u[UNR];
        if (full && s0 + UNR <= steps) {
#pragma unroll
            for (int i = 0; i < UNR; ++i) u[i] = __ldg(src + static_cast<long long>(r0 + (s0 + i) * RPI) * VPR + vec);
        } else {
#pragma unroll
            for (int i = 0; i < UNR; ++i) {
                const int r = r0 + (s0 + i) * RPI;
                bool take = s0 + i < steps;
                if (take && !full) {
                    const int ox = r % g.tw, oy = (r / g.tw) % g.th, of = r / (g.tw * g.th);
                    take = of < nf && oy < ny && ox < nx;
                }
                u[i] = take ? __ldg(src + static_cast<long long>(r) * VPR + vec) : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int i = 0; i < UNR; ++i) pool_add(acc2, u[i]);
    }
    pool_write<D>(acc2, lane, nf * ny * nx, (bh * g.nb + blk) * D, is_k, out);
}

// Reorder and pooling in one pass over raster Q and K.  One warp per (tensor,
// b, block, h) unit, h fastest, so the warps running at one time read every
// head of the same raster tokens (contiguous H * D runs) instead of one
// 2*D-byte row every H * 2*D bytes.  The warp copies the block's bs raster rows into
// its tile, 32 tile rows a round (padding rows written as zeros), and adds
// each loaded vector to its pair sums.  Lane l always holds column slice
// l % (D/8) and meets its rows in increasing order, exactly as in
// pool_kernel, so the means are bit-identical to pooling the tiles after a
// separate reorder.  Two CTAs per SM (at most 128 registers a thread) keep
// 16 warps x 8 KB of loads in flight per SM; one CTA (the unbounded
// allocation) halves that and the bandwidth with it.
template <int D>
__global__ void __launch_bounds__(256, 2) reorder_pool_kernel(Geo g, const uint4* __restrict__ q,
                                                           const uint4* __restrict__ k, uint4* __restrict__ qt,
                                                           uint4* __restrict__ kt, PoolOut out) {
    constexpr int VPR = D / 8;             // 16-byte vectors per row
    constexpr int RPI = 32 / VPR;          // rows per warp instruction
    pdl_launch_dependents();   // the score kernel may be scheduled as this grid drains
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long unit = static_cast<long long>(blockIdx.x) * 8 + warp;
    const long long per_tensor = static_cast<long long>(g.B) * g.H * g.nb;
    if (unit >= 2 * per_tensor) return;
    const bool is_k = unit >= per_tensor;
    const long long ub = is_k ? unit - per_tensor : unit;
    const int h = static_cast<int>(ub % g.H);
    const long long bblk = ub / g.H;                       // b * nb + block
    const int blk = static_cast<int>(bblk % g.nb);
    const int b = static_cast<int>(bblk / g.nb);
    const long long bh = static_cast<long long>(b) * g.H + h;
    const uint4* src = is_k ? k : q;
    uint4* dst = (is_k ? kt : qt) + (bh * g.Npad + static_cast<long long>(blk) * g.bs) * VPR;
    const int tile = tile_of_block(g, blk);
    const int bx = tile % g.nbx, by = (tile / g.nbx) % g.nby, bf = tile / (g.nbx * g.nby);
    const int nf = min(g.tf, g.F - bf * g.tf);
    const int ny = min(g.th, g.Hs - by * g.th);
    const int nx = min(g.tw, g.Ws - bx * g.tw);
    const int vec = lane % VPR;
    unsigned long long acc2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) acc2[e] = 0ull;
    for (int r32 = 0; r32 < g.bs; r32 += 32) {
        // raster row of tile row r32 + lane, or -1 (padding, or past the tile when bs = 16)
        long long s_row = -1;
        const int o = r32 + lane;
        if (o < g.bs) {
            const int ox = o % g.tw, oy = (o / g.tw) % g.th, of = o / (g.tw * g.th);
            if (of < nf && oy < ny && ox < nx) {
                const long long n =
                    (static_cast<long long>(bf * g.tf + of) * g.Hs + by * g.th + oy) * g.Ws + bx * g.tw + ox;
                s_row = (static_cast<long long>(b) * g.N + n) * g.H + h;
            }
        }
        uint4 v[VPR];   // 32 rows x VPR vectors over 32 lanes, all in flight
#pragma unroll
        for (int it = 0; it < VPR; ++it) {
            const long long sr = __shfl_sync(0xffffffffu, s_row, it * RPI + lane / VPR);
            v[it] = sr >= 0 ? __ldg(src + sr * VPR + vec) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int it = 0; it < VPR; ++it) {
            const int r = r32 + it * RPI + lane / VPR;
            if (r < g.bs) dst[static_cast<long long>(r) * VPR + vec] = v[it];
            pool_add(acc2, v[it]);
        }
    }
    pool_write<D>(acc2, lane, nf * ny * nx, (bh * g.nb + blk) * D, is_k, out);
}

// ------------------------------------------------------------------ scoring

// L = scale * Qp Kp^T per (b, h) on the tensor cores, in three tf32 products:
// with x = x_hi + x_lo (x_hi the tf32 part), Qp Kp^T is taken as
// hi*hi + hi*lo + lo*hi, which leaves only the lo*lo term (2^-22 relative)
// out, close to an fp32 product.  A tile is 128 query blocks x 256 key
// blocks; its accumulator lives in TMEM (256 fp32 columns, two tiles in
// flight).  Persistent CTAs, warp-specialised:
//   warp 0      TMA producer: per 32-wide slice of the head dimension, the
//               hi and lo parts of the Q rows and the K rows (96 KB a stage,
//               two stages), 128-byte swizzled, K-major.
//   warp 1      TMEM owner and MMA issuer: 4 x 3 MMAs (M=128, N=256, K=8) a
//               slice; a commit frees the stage, the tile's last commit hands
//               the accumulator to the epilogue.
//   warps 2-5   epilogue: each thread owns one query-block row of the tile
//               (the warp's TMEM lane quarter), reads 32 columns at a time
//               and scales them.  When rows are 16-byte multiples (nb % 4 ==
//               0) a warp stages its 32 x 32 block in shared memory (128-byte
//               swizzle, two buffers) and writes it with one TMA store into
//               the [B*H, nb, nb] logits, which clips rows and columns past
//               nb; otherwise threads store their real logits directly.
constexpr int SC_BM = 128;                 // query blocks per tile (MMA M)
constexpr int SC_BN = 256;                 // key blocks per tile (MMA N)
constexpr int SC_SLICE = 32;               // fp32 head-dim elements per stage (128 bytes)
constexpr int SC_STAGES = 2;
constexpr int SC_THREADS = 192;
constexpr uint32_t SC_A_BYTES = SC_BM * 128u;
constexpr uint32_t SC_B_BYTES = SC_BN * 128u;
constexpr uint32_t SC_STAGE_BYTES = 2u * SC_A_BYTES + 2u * SC_B_BYTES;
constexpr uint32_t SC_TMEM_COLS = 2u * SC_BN;
constexpr uint32_t SC_OUT_BYTES = 32u * 128u;   // one warp's 32 x 32 fp32 staging block

struct ScoreCtrl {
    unsigned long long full[SC_STAGES];
    unsigned long long empty[SC_STAGES];
    unsigned long long acc_full[2];
    unsigned long long acc_empty[2];
    unsigned long long drained;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr uint32_t SC_OUT_OFF = SC_STAGES * SC_STAGE_BYTES;            // 4 warps x 2 buffers
constexpr uint32_t SC_CTRL_OFF = SC_OUT_OFF + 8u * SC_OUT_BYTES;
constexpr uint32_t SC_SMEM = SC_CTRL_OFF + static_cast<uint32_t>(sizeof(ScoreCtrl));
static_assert(SC_SMEM <= 232448u, "score kernel shared memory");

struct ScoreArgs {
    float* L;
    float scale;
    int nb;
    int m_tiles, n_tiles;
    int slices;            // D / 32
    int tma_out;           // logits stored through t_out (nb % 4 == 0)
    long long tiles;       // B*H * m_tiles * n_tiles
};

__global__ void __launch_bounds__(SC_THREADS, 1) score_kernel(const __grid_constant__ CUtensorMap tq_hi,
                                                              const __grid_constant__ CUtensorMap tq_lo,
                                                              const __grid_constant__ CUtensorMap tk_hi,
                                                              const __grid_constant__ CUtensorMap tk_lo,
                                                              const __grid_constant__ CUtensorMap t_out,
                                                              ScoreArgs a) {
    extern __shared__ __align__(1024) unsigned char sc_smem[];
    ScoreCtrl& ctl = *reinterpret_cast<ScoreCtrl*>(sc_smem + SC_CTRL_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &ctl.abort_flag;
    if (threadIdx.x == 0) {
        if ((smem_u32(sc_smem) & 1023u) != 0u) record_status(FVATTN_ERR_BOUNDS);
        for (int s = 0; s < SC_STAGES; ++s) {
            mbar_init(smem_u32(&ctl.full[s]), 1);
            mbar_init(smem_u32(&ctl.empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&ctl.acc_full[b]), 1);
            mbar_init(smem_u32(&ctl.acc_empty[b]), 128);
        }
        mbar_init(smem_u32(&ctl.drained), 1);
        ctl.abort_flag = (smem_u32(sc_smem) & 1023u) != 0u;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl.tmem_base), SC_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    const int per_head = a.m_tiles * a.n_tiles;
    pdl_launch_dependents();   // the select kernel may be scheduled as this grid drains
    pdl_wait();                // pooled Q/K of the previous kernel complete and visible

    if (warp == 0) {
        // ---- TMA producer
        if (lane == 0 && !*abort_flag) {
            prefetch_tmap(&tq_hi);
            prefetch_tmap(&tq_lo);
            prefetch_tmap(&tk_hi);
            prefetch_tmap(&tk_lo);
            long long seq = 0;
            for (long long t = blockIdx.x; t < a.tiles; t += gridDim.x) {
                const long long bh = t / per_head;
                const int rem = static_cast<int>(t - bh * per_head);
                const int qrow = static_cast<int>(bh * a.nb) + (rem / a.n_tiles) * SC_BM;
                const int krow = static_cast<int>(bh * a.nb) + (rem % a.n_tiles) * SC_BN;
                bool ok = true;
                for (int ks = 0; ks < a.slices; ++ks, ++seq) {
                    const int s = static_cast<int>(seq % SC_STAGES);
                    if (!wait_bar(smem_u32(&ctl.empty[s]), ((seq / SC_STAGES) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t base = smem_u32(sc_smem + s * SC_STAGE_BYTES);
                    const uint32_t fb = smem_u32(&ctl.full[s]);
                    mbar_arrive_expect_tx(fb, SC_STAGE_BYTES);
                    tma_load_2d(base, &tq_hi, ks * SC_SLICE, qrow, fb);
                    tma_load_2d(base + SC_A_BYTES, &tq_lo, ks * SC_SLICE, qrow, fb);
                    tma_load_2d(base + 2 * SC_A_BYTES, &tk_hi, ks * SC_SLICE, krow, fb);
                    tma_load_2d(base + 2 * SC_A_BYTES + SC_B_BYTES, &tk_lo, ks * SC_SLICE, krow, fb);
                }
                if (!ok) break;
            }
            // copies still in flight finish before the CTA can exit
            for (long long q = seq > SC_STAGES ? seq - SC_STAGES : 0; q < seq; ++q)
                wait_bar_drain(smem_u32(&ctl.full[q % SC_STAGES]), (q / SC_STAGES) & 1);
        }
    } else if (warp == 1) {
        // ---- MMA issuer
        if (lane == 0 && !*abort_flag) {
            constexpr uint32_t idesc = idesc_tf32_f32(SC_BM, SC_BN);
            long long seq = 0, tcount = 0;
            for (long long t = blockIdx.x; t < a.tiles; t += gridDim.x, ++tcount) {
                const int b = static_cast<int>(tcount & 1);
                if (!wait_bar(smem_u32(&ctl.acc_empty[b]), ((tcount >> 1) & 1) ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(b * SC_BN);
                bool ok = true;
                for (int ks = 0; ks < a.slices; ++ks, ++seq) {
                    const int s = static_cast<int>(seq % SC_STAGES);
                    if (!wait_bar(smem_u32(&ctl.full[s]), (seq / SC_STAGES) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t base = smem_u32(sc_smem + s * SC_STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < SC_SLICE / 8; ++kk) {
                        const uint32_t off = kk * 32u;   // 8 tf32 = 32 bytes inside the swizzle atom
                        const uint64_t ah = sw128_desc(base + off, 16, 1024);
                        const uint64_t al = sw128_desc(base + SC_A_BYTES + off, 16, 1024);
                        const uint64_t bhd = sw128_desc(base + 2 * SC_A_BYTES + off, 16, 1024);
                        const uint64_t bld = sw128_desc(base + 2 * SC_A_BYTES + SC_B_BYTES + off, 16, 1024);
                        mma_tf32_ss(d, ah, bhd, idesc, (ks | kk) != 0);
                        mma_tf32_ss(d, ah, bld, idesc, 1u);
                        mma_tf32_ss(d, al, bhd, idesc, 1u);
                    }
                    mma_commit(smem_u32(&ctl.empty[s]));
                }
                if (!ok) break;
                mma_commit(smem_u32(&ctl.acc_full[b]));
            }
            // MMAs still in flight finish before TMEM is released
            mma_commit(smem_u32(&ctl.drained));
            wait_bar_drain(smem_u32(&ctl.drained), 0);
        }
    } else {
        // ---- epilogue: thread = one query-block row of the tile
        const int quarter = warp & 3;
        const int r_in = quarter * 32 + lane;
        const bool vec_ok = (a.nb & 3) == 0;
        const uint32_t stage0 = smem_u32(sc_smem + SC_OUT_OFF + static_cast<uint32_t>(quarter) * 2u * SC_OUT_BYTES);
        if (lane == 0 && a.tma_out) prefetch_tmap(&t_out);
        long long tcount = 0;
        int nstore = 0;
        for (long long t = blockIdx.x; t < a.tiles; t += gridDim.x, ++tcount) {
            const int b = static_cast<int>(tcount & 1);
            if (!wait_warp(smem_u32(&ctl.acc_full[b]), (tcount >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const long long bh = t / per_head;
            const int rem = static_cast<int>(t % per_head);
            const int row0 = (rem / a.n_tiles) * SC_BM;
            const int row = row0 + r_in;
            const int col0 = (rem % a.n_tiles) * SC_BN;
            float* out = a.L + (bh * a.nb + row) * static_cast<long long>(a.nb);
            const bool row_ok = row < a.nb;
            for (int c = 0; c < SC_BN; c += 32) {
                const int col = col0 + c;
                if (col >= a.nb) break;
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * SC_BN + c), r);
                tmem_wait_ld();
                if (a.tma_out) {
                    // swizzled staging: 16-byte chunk j of row `lane` at chunk j ^ (lane & 7)
                    const uint32_t buf = stage0 + static_cast<uint32_t>(nstore & 1) * SC_OUT_BYTES;
                    if (lane == 0) bulk_wait_group_read<1>();   // this buffer's previous store has read it
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t dst = buf + static_cast<uint32_t>(lane) * 128u +
                                             static_cast<uint32_t>((j ^ (lane & 7)) * 16);
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                                     "f"(__uint_as_float(r[4 * j]) * a.scale),
                                     "f"(__uint_as_float(r[4 * j + 1]) * a.scale),
                                     "f"(__uint_as_float(r[4 * j + 2]) * a.scale),
                                     "f"(__uint_as_float(r[4 * j + 3]) * a.scale)
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&t_out, buf, col, row0 + quarter * 32, static_cast<int>(bh));
                        bulk_commit_group();
                    }
                    ++nstore;
                } else if (row_ok && vec_ok && col + 32 <= a.nb) {
                    float4* o4 = reinterpret_cast<float4*>(out + col);
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        o4[v] = make_float4(__uint_as_float(r[4 * v]) * a.scale, __uint_as_float(r[4 * v + 1]) * a.scale,
                                            __uint_as_float(r[4 * v + 2]) * a.scale,
                                            __uint_as_float(r[4 * v + 3]) * a.scale);
                } else if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (col + i < a.nb) out[col + i] = __uint_as_float(r[i]) * a.scale;
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&ctl.acc_empty[b]));
        }
        // logits stores complete before the kernel ends
        if (lane == 0 && a.tma_out) bulk_wait_group_all();
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, SC_TMEM_COLS);
}

// ------------------------------------------------------------------ selection

constexpr int SEL_WARPS = 8;
constexpr int SEL_VALUE_STEPS = 16;   // value-midpoint steps before key-space bisection

// Monotone 32-bit key of a float: a < b  <=>  fkey(a) < fkey(b).  -0 is
// folded into +0 first, so equal logits get equal keys.
__device__ __forceinline__ uint32_t fkey(float v) {
    const uint32_t b = __float_as_uint(v + 0.0f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Order key of (logit, index): ascending key = logit descending, then index
// ascending.
__device__ __forceinline__ unsigned long long order_key(float v, int j) {
    return (static_cast<unsigned long long>(~fkey(v)) << 32) | static_cast<uint32_t>(j);
}

// Masses are fixed point with 40 fractional bits: a lane's float partial sum
// (at most 80 entries of exp(l - lmax) <= 1) converts exactly, and the warp
// sum of those integers is the same on every lane whatever the order.
constexpr float SEL_FIX = 1099511627776.0f;   // 2^40

// Sum over the row of [v >= t] * e (fixed point) and of [v >= t].
template <int NPL, bool KEEP_E>
__device__ __forceinline__ void sel_eval(const float (&v)[NPL], const float (&e)[NPL], float lmax, float t,
                                         bool mass, unsigned long long& s, int& c) {
    float m0 = 0.f, m1 = 0.f;
    int n = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const bool in = v[i] >= t;
        n += in;
        if (mass) {
            const float x = KEEP_E ? e[i] : __expf(v[i] - lmax);
            if (in) {
                if (i & 1) m1 += x;
                else m0 += x;
            }
        }
    }
    c = __reduce_add_sync(0xffffffffu, static_cast<unsigned int>(n));
    if (mass) {
        unsigned long long f = static_cast<unsigned long long>((m0 + m1) * SEL_FIX);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
        s = f;
    } else {
        s = static_cast<unsigned long long>(c);
    }
}

// Boundary of a weighted prefix in (logit desc, index asc) order: the first
// entry at which the running weight reaches `target`, where the weight of the
// set {v >= t} is sel_eval's sum (mass) or count.  Precondition:
// weight({v >= lmin}) >= target > 0, c_all = #{v >= lmin}.  The bracket [lo, hi) in key
// space always holds the crossing (weight at lo >= target > weight at hi); it
// is halved at the value midpoint for the first steps, then at the key
// midpoint, until at most 32 entries remain (sorted and scanned by one warp)
// or a single logit value remains (ties resolved by ascending index).
// Returns the crossing's order key and its 1-based rank.
template <int NPL, bool KEEP_E>
__device__ unsigned long long sel_boundary(const float (&v)[NPL], const float (&e)[NPL], float lmax, float lmin,
                                           bool mass, int c_all, double target,
                                           unsigned long long* ck, int* rank) {
    const int lane = threadIdx.x & 31;
    uint32_t lo_k = fkey(lmin), hi_k = fkey(lmax) + 1u;
    unsigned long long s_hi = 0ull;
    int c_lo = c_all, c_hi = 0;
#pragma unroll 1
    for (int it = 0; c_lo - c_hi > 32 && hi_k - lo_k > 1u; ++it) {
        uint32_t mk;
        if (it < SEL_VALUE_STEPS) {
            const float a = key_to_float(lo_k), b = key_to_float(hi_k - 1u);
            mk = fkey(0.5f * a + 0.5f * b);
        } else {
            mk = lo_k + (hi_k - lo_k) / 2u;
        }
        mk = min(max(mk, lo_k + 1u), hi_k - 1u);
        unsigned long long s;
        int c;
        sel_eval<NPL, KEEP_E>(v, e, lmax, key_to_float(mk), mass, s, c);
        if (static_cast<double>(s) >= target) {
            lo_k = mk;
            c_lo = c;
        } else {
            hi_k = mk;
            s_hi = s;
            c_hi = c;
        }
    }
    const float tlo = key_to_float(lo_k), thi = key_to_float(hi_k);
    const int cand = c_lo - c_hi;
    if (cand <= 32) {
        // gather the candidates, sort by order key, scan their weights
        int seen = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const bool in = v[i] >= tlo && v[i] < thi;
            const unsigned int bal = __ballot_sync(0xffffffffu, in);
            if (in) ck[seen + __popc(bal & ((1u << lane) - 1u))] = order_key(v[i], lane + 32 * i);
            seen += __popc(bal);
        }
        __syncwarp();
        unsigned long long key = lane < cand ? ck[lane] : ~0ull;
        __syncwarp();
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                const unsigned long long ok = __shfl_xor_sync(0xffffffffu, key, stride);
                const bool up = ((lane & size) == 0) == ((lane & stride) == 0);
                if (up ? (ok < key) : (ok > key)) key = ok;
            }
        }
        int pick;
        if (mass) {
            const float x = key_to_float(~static_cast<uint32_t>(key >> 32));
            unsigned long long pre = lane < cand ? static_cast<unsigned long long>(__expf(x - lmax) * SEL_FIX) : 0ull;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long t = __shfl_up_sync(0xffffffffu, pre, o);
                if (lane >= o) pre += t;
            }
            const unsigned int bal =
                __ballot_sync(0xffffffffu, lane < cand && static_cast<double>(s_hi + pre) >= target);
            pick = bal ? __ffs(bal) - 1 : cand - 1;   // rounding: all candidates
        } else {
            pick = static_cast<int>(target) - c_hi - 1;
        }
        pick = min(max(pick, 0), cand - 1);
        *rank = c_hi + pick + 1;
        return __shfl_sync(0xffffffffu, key, pick);
    }
    // a single logit value remains: take the candidates by ascending index
    long long need;
    if (mass) {
        const double w = static_cast<double>(static_cast<unsigned long long>(__expf(tlo - lmax) * SEL_FIX));
        need = w > 0.0 ? static_cast<long long>(ceil((target - static_cast<double>(s_hi)) / w)) : cand;
    } else {
        need = static_cast<long long>(target) - c_hi;
    }
    need = min(max(need, 1ll), static_cast<long long>(cand));
    int seen = 0, found = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const bool in = v[i] == tlo;
        const unsigned int bal = __ballot_sync(0xffffffffu, in);
        if (in && seen + __popc(bal & ((1u << lane) - 1u)) + 1 == need) found = lane + 32 * i + 1;
        seen += __popc(bal);
    }
    found = __reduce_max_sync(0xffffffffu, static_cast<unsigned int>(found));
    *rank = c_hi + static_cast<int>(need);
    return order_key(tlo, found - 1);
}

// One warp per (b, h, query block) row.  Kept set: the first m entries of the
// order, m = min(nb, max(m_p, min(k, nb)) + kextra), m_p the Top-p crossing
// (first prefix whose mass reaches p * total; 0 when p = 0, nb when p >= 1).
template <int NPL, bool KEEP_E>
__global__ void __launch_bounds__(32 * SEL_WARPS, NPL <= 24 ? 4 : 1) select_kernel(int nb, long long rows, const float* __restrict__ L,
                                                                double p, int kfloor, int kextra,
                                                                int32_t* __restrict__ kv_idx,
                                                                int32_t* __restrict__ kv_cnt) {
    __shared__ unsigned long long cand_keys[SEL_WARPS][32];
    pdl_wait();                // logits of the score kernel complete and visible
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * SEL_WARPS + warp;
    if (row >= rows) return;
    const float* Lr = L + row * nb;
    float v[NPL];
    float lmax = -INFINITY, lmin = INFINITY;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int j = lane + 32 * i;
        v[i] = j < nb ? Lr[j] + 0.0f : -INFINITY;
        lmax = fmaxf(lmax, v[i]);
        if (j < nb) lmin = fminf(lmin, v[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        lmin = fminf(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
    }
    const int kf = min(kfloor, nb);
    unsigned long long thr = ~0ull;
    if (p < 1.0) {
        float e[NPL];
        if (KEEP_E) {
#pragma unroll
            for (int i = 0; i < NPL; ++i) e[i] = __expf(v[i] - lmax);
        }
        unsigned long long s_all;
        int c_all;
        int rank = 0;   // m_p
        if (p > 0.0) {
            sel_eval<NPL, KEEP_E>(v, e, lmax, lmin, true, s_all, c_all);
            const double target = p * static_cast<double>(s_all);
            thr = sel_boundary<NPL, KEEP_E>(v, e, lmax, lmin, true, c_all, target, cand_keys[warp], &rank);
        } else {
            sel_eval<NPL, KEEP_E>(v, e, lmax, lmin, false, s_all, c_all);
        }
        // floor and augmentation: the want-th entry of the order, if later
        const long long want = min(static_cast<long long>(nb), static_cast<long long>(max(rank, kf)) + kextra);
        if (want >= c_all) {
            thr = ~0ull;
        } else if (want > rank) {
            thr = sel_boundary<NPL, KEEP_E>(v, e, lmax, lmin, false, c_all, static_cast<double>(want),
                                            cand_keys[warp], &rank);
        }
    }
    // emit the kept indices in ascending order
    const float tv = key_to_float(~static_cast<uint32_t>(thr >> 32));
    const int tj = static_cast<int>(thr & 0xffffffffu);
    const bool all = thr == ~0ull;
    int32_t* out = kv_idx + row * nb;
    int written = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int j = lane + 32 * i;
        const bool keep = j < nb && (all || v[i] > tv || (v[i] == tv && j <= tj));
        const unsigned int bal = __ballot_sync(0xffffffffu, keep);
        if (keep) out[written + __popc(bal & ((1u << lane) - 1u))] = j;
        written += __popc(bal);
    }
    if (lane == 0) kv_cnt[row] = written;
}

template <int NPL, bool KEEP_E>
static int launch_select(long long rows, int nb, const float* L, double p, int kfloor, int kextra, int32_t* kv_idx,
                         int32_t* kv_cnt, cudaStream_t s) {
    const long long blocks = (rows + SEL_WARPS - 1) / SEL_WARPS;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(32 * SEL_WARPS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, select_kernel<NPL, KEEP_E>, nb, rows, L, p, kfloor, kextra, kv_idx, kv_cnt) !=
        cudaSuccess)
        return FVATTN_ERR_CUDA;
    FV_CHECK_LAUNCH();
    return FVATTN_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace: tf32 hi / lo parts of the pooled Q and K ([B*H*nb, D] fp32
// each), then the logits ([B*H*nb, nb] fp32).
struct RouteWs {
    size_t qh, ql, kh, kl, logits, total;
};

static size_t al256(size_t x) { return (x + 255) / 256 * 256; }

static RouteWs route_ws(const fvattn_geom& g) {
    RouteWs w;
    const size_t BH = static_cast<size_t>(g.B) * g.H;
    const size_t pooled = al256(sizeof(float) * BH * g.nb * g.D);
    w.qh = 0;
    w.ql = pooled;
    w.kh = 2 * pooled;
    w.kl = 3 * pooled;
    w.logits = 4 * pooled;
    w.total = w.logits + al256(sizeof(float) * BH * g.nb * g.nb);
    return w;
}

static int score_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

}  // namespace fv

using namespace fv;

extern "C" size_t fvattn_route_workspace_size(const fvattn_geom* gp) {
    if (!gp) return 0;
    return route_ws(*gp).total;
}

extern "C" int fvattn_route_kernel_launches(const fvattn_geom* gp) {
    if (!gp || gp->B <= 0 || gp->H <= 0) return 0;
    return 3;   // pool, score, select
}

// Pooling (from the tiles, or fused with the reorder when raster Q and K are
// given, which then writes the tiles), scoring and selection.
static int route_impl(const fvattn_geom* gp, const void* q_raster, const void* k_raster, const void* q_tiled,
                      const void* k_tiled, double p, int k_floor, int k_extra, float scale, int32_t* kv_idx,
                      int32_t* kv_cnt, float* q_pool, float* k_pool, float* logits, void* workspace,
                      size_t ws_bytes, fvattn_stream_t stream) {
    if (!gp || !q_tiled || !k_tiled || !kv_idx || !kv_cnt) return FVATTN_ERR_INVALID;
    if (!aligned16(q_tiled) || !aligned16(k_tiled) || !aligned16(kv_idx) || !aligned16(kv_cnt))
        return FVATTN_ERR_INVALID;
    const bool fused = q_raster != nullptr || k_raster != nullptr;
    if (fused && (!q_raster || !k_raster || !aligned16(q_raster) || !aligned16(k_raster) || q_tiled == k_tiled))
        return FVATTN_ERR_INVALID;
    if (!(p >= 0.0 && p <= 1.0) || k_floor < 1 || k_extra < 0 || !isfinite(scale)) return FVATTN_ERR_INVALID;
    if (gp->nb <= 0 || gp->nb > 2560) return FVATTN_ERR_UNSUPPORTED;
    if (gp->D != 64 && gp->D != 128) return FVATTN_ERR_UNSUPPORTED;
    const Geo g = to_geo(*gp);
    const RouteWs wl = route_ws(*gp);
    char* ws = static_cast<char*>(workspace);
    if (!workspace || ws_bytes < wl.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return FVATTN_ERR_INVALID;
    if ((q_pool && !aligned16(q_pool)) || (k_pool && !aligned16(k_pool)) || (logits && !aligned16(logits)))
        return FVATTN_ERR_INVALID;
    float* L = logits ? logits : reinterpret_cast<float*>(ws + wl.logits);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    PoolOut po;
    po.hi[0] = reinterpret_cast<float*>(ws + wl.qh);
    po.lo[0] = reinterpret_cast<float*>(ws + wl.ql);
    po.hi[1] = reinterpret_cast<float*>(ws + wl.kh);
    po.lo[1] = reinterpret_cast<float*>(ws + wl.kl);
    po.mean[0] = q_pool;
    po.mean[1] = k_pool;
    const long long units = 2ll * g.B * g.H * g.nb;
    const unsigned pblocks = static_cast<unsigned>((units + 7) / 8);
    if (fused) {
        const uint4 *qr = static_cast<const uint4*>(q_raster), *kr = static_cast<const uint4*>(k_raster);
        uint4 *qw = static_cast<uint4*>(const_cast<void*>(q_tiled)), *kw = static_cast<uint4*>(const_cast<void*>(k_tiled));
        if (g.D == 128)
            reorder_pool_kernel<128><<<pblocks, 256, 0, s>>>(g, qr, kr, qw, kw, po);
        else
            reorder_pool_kernel<64><<<pblocks, 256, 0, s>>>(g, qr, kr, qw, kw, po);
    } else if (g.D == 128) {
        pool_kernel<128><<<pblocks, 256, 0, s>>>(g, static_cast<const __nv_bfloat16*>(q_tiled),
                                                 static_cast<const __nv_bfloat16*>(k_tiled), po);
    } else {
        pool_kernel<64><<<pblocks, 256, 0, s>>>(g, static_cast<const __nv_bfloat16*>(q_tiled),
                                                static_cast<const __nv_bfloat16*>(k_tiled), po);
    }
    FV_CHECK_LAUNCH();

    const unsigned long long prow = static_cast<unsigned long long>(g.B) * g.H * g.nb;
    CUtensorMap tqh, tql, tkh, tkl;
    if (!make_tmap_2d(&tqh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, po.hi[0], prow, g.D, SC_SLICE, SC_BM) ||
        !make_tmap_2d(&tql, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, po.lo[0], prow, g.D, SC_SLICE, SC_BM) ||
        !make_tmap_2d(&tkh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, po.hi[1], prow, g.D, SC_SLICE, SC_BN) ||
        !make_tmap_2d(&tkl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, po.lo[1], prow, g.D, SC_SLICE, SC_BN))
        return FVATTN_ERR_CUDA;
    ScoreArgs sa;
    sa.L = L;
    sa.scale = scale;
    sa.nb = g.nb;
    sa.m_tiles = (g.nb + SC_BM - 1) / SC_BM;
    sa.n_tiles = (g.nb + SC_BN - 1) / SC_BN;
    sa.slices = g.D / SC_SLICE;
    sa.tma_out = (g.nb % 4) == 0;
    CUtensorMap tout;
    std::memset(&tout, 0, sizeof(tout));
    if (sa.tma_out &&
        !make_tmap_3d(&tout, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, L, static_cast<unsigned long long>(g.B) * g.H, g.nb,
                      g.nb, 1, 32, 32))
        return FVATTN_ERR_CUDA;
    sa.tiles = static_cast<long long>(g.B) * g.H * sa.m_tiles * sa.n_tiles;
    const int nsm = score_sms();
    if (nsm <= 0) return FVATTN_ERR_CUDA;
    if (cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(SC_SMEM)) !=
        cudaSuccess)
        return FVATTN_ERR_CUDA;
    const unsigned sgrid = static_cast<unsigned>(sa.tiles < nsm ? sa.tiles : nsm);
    {
        // programmatic serialisation: the kernel is scheduled while pooling drains and waits in-kernel
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3(sgrid);
        cfg.blockDim = dim3(SC_THREADS);
        cfg.dynamicSmemBytes = SC_SMEM;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, score_kernel, tqh, tql, tkh, tkl, tout, sa) != cudaSuccess) return FVATTN_ERR_CUDA;
    }
    FV_CHECK_LAUNCH();
    const long long rows = static_cast<long long>(g.B) * g.H * g.nb;
    // entries per lane: the smallest instantiated count that covers a row
    const int npl = (g.nb + 31) / 32;
    if (npl <= 4) return launch_select<4, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 8) return launch_select<8, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 10) return launch_select<10, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 12) return launch_select<12, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 16) return launch_select<16, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 21) return launch_select<21, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 24) return launch_select<24, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 32) return launch_select<32, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 40) return launch_select<40, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    if (npl <= 48) return launch_select<48, true>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
    return launch_select<80, false>(rows, g.nb, L, p, k_floor, k_extra, kv_idx, kv_cnt, s);
}

extern "C" int fvattn_route(const fvattn_geom* gp, const void* q_tiled, const void* k_tiled, double p, int k_floor,
                            float scale, int32_t* kv_idx, int32_t* kv_cnt, float* q_pool, float* k_pool,
                            float* logits, void* workspace, size_t ws_bytes, fvattn_stream_t stream) {
    if (!(p > 0.0)) return FVATTN_ERR_INVALID;
    return route_impl(gp, nullptr, nullptr, q_tiled, k_tiled, p, k_floor, 0, scale, kv_idx, kv_cnt, q_pool, k_pool,
                      logits, workspace, ws_bytes, stream);
}

extern "C" int fvattn_route_aug(const fvattn_geom* gp, const void* q_tiled, const void* k_tiled, double p,
                                int k_floor, int k_extra, float scale, int32_t* kv_idx, int32_t* kv_cnt,
                                float* q_pool, float* k_pool, float* logits, void* workspace, size_t ws_bytes,
                                fvattn_stream_t stream) {
    return route_impl(gp, nullptr, nullptr, q_tiled, k_tiled, p, k_floor, k_extra, scale, kv_idx, kv_cnt, q_pool,
                      k_pool, logits, workspace, ws_bytes, stream);
}

extern "C" int fvattn_reorder_route(const fvattn_geom* gp, const void* q, const void* k, void* q_tiled,
                                    void* k_tiled, double p, int k_floor, int k_extra, float scale, int32_t* kv_idx,
                                    int32_t* kv_cnt, float* q_pool, float* k_pool, float* logits, void* workspace,
                                    size_t ws_bytes, fvattn_stream_t stream) {
    if (!q || !k) return FVATTN_ERR_INVALID;
    return route_impl(gp, q, k, q_tiled, k_tiled, p, k_floor, k_extra, scale, kv_idx, kv_cnt, q_pool, k_pool, logits,
                      workspace, ws_bytes, stream);
}

int fv::take_status_route() { return fv::take_tu_status(); }
