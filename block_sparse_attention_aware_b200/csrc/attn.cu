// Dynamic block-sparse attention on the materialised FVAttn mask
// (paperlayer.ai summary, section 2 "Background and Related Work": dynamic
// block-sparse attention; section 3 "FVAttn Design", item "Pipeline":
// attention runs on the mask that routing materialised).
//
// Work list.  An item is (b, h, query block i) and costs kv_cnt[b,h,i] key
// blocks.  Top-p makes costs uneven across heads (section 2, item on Top-p
// producing heterogeneous workloads; section 3, "Runtime Load Balancing").
// The pages balance that across GPUs by migrating heads; on one GPU the
// analogue used here is a persistent kernel with one CTA per SM that takes
// items from a shared counter in a fixed order: heads by total cost,
// heaviest first, and inside a head query blocks longest first.  Taking
// items dynamically in that order is a longest-processing-time greedy, and
// keeping concurrent items inside one head keeps that head's K/V in L2.
//
// Kernel per CTA (384 threads, one CTA per SM):
//   warp 0      K producer: takes items, TMA-loads the Q tile and, per chunk
//               of 128 keys, the selected K blocks into a 2- or 3-stage ring,
//               and writes the chunk's key-validity mask (padding tokens)
//   warp 2      V producer: the same chunks' V blocks into a 2-stage ring
//   warp 1      one lane issues S = Q K^T (tcgen05.mma, bf16 -> fp32 TMEM)
//   warp 3      one lane issues O += P V; two issuing threads keep the tensor
//               pipe busy while either waits on a barrier
//   warps 4..11 softmax, two groups of four warps: chunk c goes to group
//               c & 1, which owns S_(c&1) and O_(c&1) in TMEM and a P tile in
//               shared memory.  One query row per thread (its TMEM lane);
//               online softmax in fp32 from registers (the whole S row is
//               loaded and S_w released at once; exp2 on the MUFU; eight
//               independent max and sum chains); P rounded to bf16 in the
//               128-byte-swizzled K-major layout; a chunk is computed against
//               the running reference maximum and redone, with O rescaled,
//               only when a row sum passes RESCALE_SUM_LIMIT.  At the end of
//               an item the groups swap (m, l) per row and each writes half
//               of the output columns.
// Query groups (bs < 128): one 128-row tile holds G = 128 / bs consecutive
// query blocks (their rows are contiguous in the tiled layout), so the MMA
// tile is never half empty.  The tile walks the union of the G kv lists in
// ascending block order, read from a union list (block ids with their
// membership bits) that group_union_kernel writes once per launch, so the
// loading warps do no set arithmetic per chunk; each chunk carries one key
// mask per query block of the tile, so a row only sees the keys of its own
// block's list.
// Every wait is bounded; a wait that runs out records FVATTN_ERR_TIMEOUT,
// raises a CTA-wide abort flag and all roles leave their loops, so the CTA
// always reaches the TMEM release.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "ptx.cuh"
#include "sync.cuh"
#include "tmap.cuh"

namespace fv {

constexpr int SOFTMAX_WARPS = 8;        // two groups of four warps
constexpr int FIRST_SOFTMAX_WARP = 4;   // warps 0..3: K producer, QK issuer, V producer, PV issuer
constexpr int ATT_THREADS = 32 * (FIRST_SOFTMAX_WARP + SOFTMAX_WARPS);
constexpr int MAX_K_STAGES = 3;         // K ring: a stage is free once its S = Q K^T is done
constexpr int V_STAGES = 2;             // V ring: a stage is free once its O += P V is done
constexpr uint32_t MAX_DYN_SMEM = 232448;   // sm_100 opt-in shared memory per block
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t O_COL = 256;          // S_w at columns 128*w, O_w at 256 + 128*w
// Lazy rescaling: after an item's first chunk, a chunk's P is computed against
// the running reference maximum without looking at the chunk's own maximum;
// only when a row's chunk sum exceeds this (so some P may be large) is the
// chunk redone against its exact maximum with O rescaled.  P below 2^30 is
// held by bf16 P (8-bit exponent) and fp32 sums with their usual relative
// precision.
constexpr float RESCALE_SUM_LIMIT = 1073741824.0f;   // 2^30
constexpr int MAX_GROUP = 8;             // query blocks per tile at bs = 16
// Register split: the launch gives every thread LAUNCH_REGS; the producer and
// issuer warpgroup drops to RegSplit::LOW and the two softmax warpgroups
// (which hold a whole 128-column S row) rise to RegSplit::HIGH.  One
// warpgroup at LOW plus two at HIGH must fit in what the CTA was launched
// with; the host checks the compiled register count before every launch.
// The softmax computes half of a chunk's exponentials before it needs P_w,
// which takes more live registers there.
constexpr int LAUNCH_REGS = 168;          // 65536 / 384 rounded down to a multiple of 8
template <bool GRP> struct RegSplit {
    static constexpr int LOW = 72;
    static constexpr int HIGH = 216;
    static_assert(128 * LOW + 256 * HIGH <= ATT_THREADS * LAUNCH_REGS, "register split");
};

struct AttnArgs {
    Geo g;
    const int32_t* kv_idx;
    const int32_t* kv_cnt;
    // Query groups: G = 128 / bs consecutive query blocks share one 128-row
    // tile.  For G > 1 an item is (b*h, group) and walks the union of the
    // group's kv lists in ascending block order.
    int G;                       // query blocks per tile (1 when bs = 128)
    int ngroups;                 // ceil(nb / G)
    const uint32_t* ulist;       // [B*H][ngroups][nb] union lists (G > 1): block | membership bits << 24
    const int32_t* gcnt;         // [B*H][ngroups] union sizes (G > 1)
    const int32_t* ext;          // [nb] real extent of each block, packed as block_extent
    const int32_t* head_order;   // [B*H] heads, heaviest first
    const int32_t* item_order;   // [B*H][nb] query blocks of each head, longest first
    int* counter;                // next item to hand out
    __nv_bfloat16* o;            // [B, H, Npad, D], or [B, N, H, D] when raster
    int raster;                  // write O rows straight to the raster layout (real tokens only)
    unsigned long long* sm_stats;
    float scale_log2;            // scale * log2(e), > 0
    int total_items;
    unsigned long long wait_limit_ns;   // bound of every wait (fault-injection tests shorten it)
    int hooks;                   // FVATTN_HOOK_* fault injection (0 in normal use)
};

struct __align__(16) Ctrl {
    unsigned long long q_full, q_empty;
    unsigned long long k_full[MAX_K_STAGES], k_empty[MAX_K_STAGES];
    unsigned long long v_full[V_STAGES], v_empty[V_STAGES];
    unsigned long long s_full[2], s_free[2];   // per softmax group w: S_w written / read
    unsigned long long p_full[2], p_free[2];   // per group: P_w written / its PV done
    unsigned long long o_free;                 // both O accumulators read by the epilogue
    unsigned long long mrg_full, mrg_empty;    // end-of-item exchange of (m, l)
    unsigned long long item_full[2], item_empty[2];
    unsigned long long blocks_done;
    unsigned long long drain[2];               // issuers' final commit: their MMAs have completed
    int item[2][4];              // bh, first query block, cnt (kv blocks to walk), valid
    uint32_t mask[MAX_K_STAGES][MAX_GROUP][4];  // per query block of the tile: its valid keys of a K stage's chunk
    uint32_t tmem_base;
    int abort_flag;
    float mrg_m[2][128];         // [group][row] running maximum (log2 units)
    float mrg_l[2][128];         // [group][row] running sum
};

template <int D>
struct Smem {
    static constexpr uint32_t Q_BYTES = 128u * D * 2u;   // D/64 halves of 16 KB
    static constexpr uint32_t KV_BYTES = 128u * D * 2u;
    static constexpr uint32_t P_BYTES = 128u * 128u * 2u; // one P tile per softmax group
    static constexpr uint32_t base_total(int ks) {
        return Q_BYTES + (ks + V_STAGES) * KV_BYTES + 2 * P_BYTES + static_cast<uint32_t>(sizeof(Ctrl));
    }
    // K ring depth: 3 stages when they fit, else 2.
    static constexpr int KS = base_total(3) <= MAX_DYN_SMEM ? 3 : 2;
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t K_OFF = Q_OFF + Q_BYTES;
    static constexpr uint32_t V_OFF = K_OFF + KS * KV_BYTES;
    static constexpr uint32_t P_OFF = V_OFF + V_STAGES * KV_BYTES;
    static constexpr uint32_t CTRL_OFF = P_OFF + 2 * P_BYTES;
    static constexpr uint32_t TOTAL = CTRL_OFF + static_cast<uint32_t>(sizeof(Ctrl));
    // Dynamic shared memory starts 1024-byte aligned on sm_100 (the kernel
    // checks); at least 120 KB so two CTAs never share an SM (each holds all
    // 512 TMEM columns).
    static constexpr uint32_t ALLOC = TOTAL > 120u * 1024u ? TOTAL : 120u * 1024u;
    static_assert(ALLOC <= MAX_DYN_SMEM, "shared-memory layout too large");
};

// Real extent of a tile: frames, rows and cols that hold tokens, packed as
// nf | ny << 8 | nx << 16 (each <= 128).
__device__ __forceinline__ int block_extent(const Geo& g, int block) {
    block = tile_of_block(g, block);
    const int bx = block % g.nbx;
    const int rest = block / g.nbx;
    const int by = rest % g.nby;
    const int bf = rest / g.nby;
    const int nf = min(g.tf, g.F - bf * g.tf);
    const int ny = min(g.th, g.Hs - by * g.th);
    const int nx = min(g.tw, g.Ws - bx * g.tw);
    return nf | (ny << 8) | (nx << 16);
}

// Block id of slot `lane` of chunk `cl` of a kv list (lanes < nblk), range-checked.
__device__ __forceinline__ int chunk_block(const int32_t* list, int cl, int bpc, int nblk, int lane, int nb) {
    int j = 0;
    if (lane < nblk) {
        j = __ldg(list + cl * bpc + lane);
        if (j < 0 || j >= nb) {
            record_status(FVATTN_ERR_BOUNDS);
            j = 0;
        }
    }
    return j;
}

// Slots of chunk cl of a query group's union list (lane s < nn: slot s):
// block id and membership bits (bit t: in the list of the tile's query
// block t), range-checked.
__device__ __forceinline__ int union_slot(const uint32_t* ul, int cl, int bpc, int nn, int lane, int nb,
                                          uint32_t& mem) {
    uint32_t e = 0u;
    if (lane < nn) e = __ldg(ul + cl * bpc + lane);
    int j = static_cast<int>(e & 0xFFFFFFu);
    mem = e >> 24;
    if (lane < nn && j >= nb) {
        record_status(FVATTN_ERR_BOUNDS);
        j = 0;
        mem = 0u;
    }
    return j;
}

// GRP: 128-row tiles of G = 128 / bs > 1 query blocks walking the union of
// their kv lists (bs < 128); otherwise one query block per tile.
template <int D, bool GRP>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
    using L = Smem<D>;
    constexpr int KS = L::KS;
    extern __shared__ __align__(1024) unsigned char smem[];
    // The 128-byte swizzle of TMA and of the tcgen05 operand descriptors
    // needs 1024-byte aligned tiles.
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) record_status(FVATTN_ERR_UNSUPPORTED);
        return;
    }
    Ctrl& ctl = *reinterpret_cast<Ctrl*>(smem + L::CTRL_OFF);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + L::Q_OFF;
    const uint32_t sK = sbase + L::K_OFF;
    const uint32_t sV = sbase + L::V_OFF;
    const uint32_t sP = sbase + L::P_OFF;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const Geo& g = a.g;
    const int bs = g.bs;
    const int bpc = 128 / bs;   // key blocks per 128-key chunk
    volatile int* abort_flag = &ctl.abort_flag;
    const unsigned long long wlim = a.wait_limit_ns;
    const unsigned long long t_start = global_timer_ns();

    // ---- set-up: zero the operand tiles (stale rows must be finite), barriers, TMEM
    {
        uint4* z = reinterpret_cast<uint4*>(smem);
        const uint32_t n16 = L::CTRL_OFF / 16u;
        for (uint32_t i = threadIdx.x; i < n16; i += ATT_THREADS) z[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&ctl.q_full), 1);
        mbar_init(smem_u32(&ctl.q_empty), 1);
        for (int s = 0; s < KS; ++s) {
            mbar_init(smem_u32(&ctl.k_full[s]), 1);
            mbar_init(smem_u32(&ctl.k_empty[s]), 1 + 4);   // QK^T commit + the owning group's mask read
        }
        for (int s = 0; s < V_STAGES; ++s) {
            mbar_init(smem_u32(&ctl.v_full[s]), 1);
            mbar_init(smem_u32(&ctl.v_empty[s]), 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(smem_u32(&ctl.s_full[w]), 1);
            mbar_init(smem_u32(&ctl.s_free[w]), 4);
            mbar_init(smem_u32(&ctl.p_full[w]), 4);
            mbar_init(smem_u32(&ctl.p_free[w]), 1);
            mbar_init(smem_u32(&ctl.item_full[w]), 1);
            mbar_init(smem_u32(&ctl.item_empty[w]), 3 + SOFTMAX_WARPS);  // two issuers, V producer, softmax
        }
        mbar_init(smem_u32(&ctl.o_free), SOFTMAX_WARPS);
        mbar_init(smem_u32(&ctl.drain[0]), 1);
        mbar_init(smem_u32(&ctl.drain[1]), 1);
        mbar_init(smem_u32(&ctl.mrg_full), SOFTMAX_WARPS);
        mbar_init(smem_u32(&ctl.mrg_empty), SOFTMAX_WARPS);
        ctl.abort_flag = 0;
        ctl.blocks_done = 0ull;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl.tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;

    if (warp >= FIRST_SOFTMAX_WARP) {
        regs_inc<RegSplit<GRP>::HIGH>();
        // =========================== softmax groups (warps 4..7: w = 0, 8..11: w = 1)
        // Group w takes the chunks c with c & 1 == w: its own S_w, P_w and
        // O_w, running maximum m and sum l.  At the end of an item the two
        // groups exchange (m, l) per row and each writes half of the output
        // columns: O = (O_0 2^(m_0-M) + O_1 2^(m_1-M)) / (l_0 2^(m_0-M) + l_1 2^(m_1-M)).
        // A chunk's whole S row is loaded into registers first and S_w is
        // released at once, so the next S = Q K^T into S_w overlaps this
        // chunk's exponentials; everything after the load works on registers.
        const int w = (warp - FIRST_SOFTMAX_WARP) >> 2;
        const int quad = warp & 3;                 // TMEM lanes 32*quad ..
        const int row = quad * 32 + lane;          // query row in the 128-row tile
        const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t sb = trow + static_cast<uint32_t>(w) * 128u;
        const uint32_t ob = trow + O_COL + static_cast<uint32_t>(w) * 128u;
        const uint32_t pbase = sP + static_cast<uint32_t>(w) * L::P_BYTES + static_cast<uint32_t>(row) * 128u;
        const int tgrp = GRP ? row / bs : 0;   // this row's query block in the tile
        const float sl2 = a.scale_log2;
        int item_seq = 0;
        uint32_t c_seq = 0;
        uint32_t n = 0;   // chunks this group has processed
        bool ok = true;
        while (ok) {
            const int slot = item_seq & 1;
            if (!wait_warp(smem_u32(&ctl.item_full[slot]), (item_seq >> 1) & 1, abort_flag, wlim)) break;
            const int bh = ctl.item[slot][0];
            const int qb = ctl.item[slot][1];
            const int cnt = ctl.item[slot][2];
            const int valid = ctl.item[slot][3];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl.item_empty[slot]));
            if (!valid) break;
            const int nc = (cnt + bpc - 1) / bpc;
            float m_ref = -INFINITY;   // reference maximum, log2 units
            float l = 0.f;
            bool mine_any = false;
            for (int cl = (static_cast<int>((c_seq + w) & 1u)); cl < nc; cl += 2) {
                // chunk c = c_seq + cl has c & 1 == w
                const uint32_t c = c_seq + cl;
                const int kst = c % KS;
                if (!wait_warp2(smem_u32(&ctl.k_full[kst]), (c / KS) & 1, smem_u32(&ctl.s_full[w]), n & 1,
                                abort_flag, wlim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // the mask words are read while the S row comes out of tensor memory
                const uint32_t* mrow = ctl.mask[kst][tgrp];
                uint32_t mw[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) mw[q] = mrow[q];
                uint32_t sv[4][32];   // this row's 128 raw scores of the chunk
#pragma unroll
                for (int q = 0; q < 4; ++q) tmem_ld32(sb + q * 32u, sv[q]);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&ctl.s_free[w]));    // S_w read: the next QK may overwrite it
                    mbar_arrive(smem_u32(&ctl.k_empty[kst]));   // mask in registers: stage free
                }
                // Exp pass: P = 2^(s*scale*log2e + negv) on fp32 pairs, row sum on fp32 pairs, bf16 P row
                // into P_w (128-byte swizzle, K-major operand).  Words whose 32 keys are all visible skip
                // the mask tests; words with none skip the exponentials.
                unsigned long long sm2[4];   // four chains of (even, odd) column sums
                // The first two quarters of the row (keys 0..63) are computed before P_w is needed, so
                // the wait for the group's previous PV to release P_w overlaps them.
                bool pw_free = false;
                auto exp_quarter = [&](int q, const unsigned long long sl2x2, const unsigned long long negx2,
                                       uint32_t (&wv)[16]) {
                    const uint32_t mword = mw[q];
                    if (mword == 0xFFFFFFFFu) {
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[q][i]), __uint_as_float(sv[q][i + 1])),
                                             sl2x2, negx2), x0, x1);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            sm2[(i >> 1) & 3] = f2_add(sm2[(i >> 1) & 3], f2_pack(p0, p1));
                            wv[i >> 1] = pack_bf16x2(p0, p1);
                        }
                    } else if (mword == 0u) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) wv[i] = 0u;
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[q][i]), __uint_as_float(sv[q][i + 1])),
                                             sl2x2, negx2), x0, x1);
                            const bool k0 = (mword >> i) & 1u, k1 = (mword >> (i + 1)) & 1u;
                            const float p0 = k0 ? ex2_approx(x0) : 0.f;
                            const float p1 = k1 ? ex2_approx(x1) : 0.f;
                            sm2[(i >> 1) & 3] = f2_add(sm2[(i >> 1) & 3], f2_pack(p0, p1));
                            wv[i >> 1] = pack_bf16x2(p0, p1);
                        }
                    }
                };
                auto store_quarter = [&](int q, const uint32_t (&wv)[16]) {
                    const int half = q >> 1;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int chunk = (((q & 1) << 2) | k4) ^ (row & 7);
                        const uint32_t addr = pbase + half * 16384u + chunk * 16u;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(wv[4 * k4]),
                                     "r"(wv[4 * k4 + 1]), "r"(wv[4 * k4 + 2]), "r"(wv[4 * k4 + 3])
                                     : "memory");
                    }
                };
                // false: the CTA aborted while waiting for P_w
                auto exp_pass = [&](float negv) -> bool {
#pragma unroll
                    for (int i = 0; i < 4; ++i) sm2[i] = 0ull;
                    const unsigned long long sl2x2 = f2_pack(sl2, sl2), negx2 = f2_pack(negv, negv);
                    uint32_t w0[16], w1[16];
                    exp_quarter(0, sl2x2, negx2, w0);
                    exp_quarter(1, sl2x2, negx2, w1);
                    if (!pw_free) {
                        if (!wait_warp(smem_u32(&ctl.p_free[w]), (n & 1) ^ 1, abort_flag, wlim)) return false;
                        pw_free = true;
                    }
                    store_quarter(0, w0);
                    store_quarter(1, w1);
                    exp_quarter(2, sl2x2, negx2, w0);
                    store_quarter(2, w0);
                    exp_quarter(3, sl2x2, negx2, w1);
                    store_quarter(3, w1);
                    return true;
                };
                auto rescale_o = [&](float alpha) {
                    tc_fence_after();
#pragma unroll 1
                    for (int q = 0; q < D / 32; ++q) {
                        uint32_t o[32];
                        tmem_ld32(ob + q * 32u, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(ob + q * 32u, o);
                    }
                    tmem_wait_st();
                };
                // Row maximum of the visible raw scores of this chunk (scaled to log2 units); -inf for a
                // row that sees no key of its block in this chunk.
                auto max_pass = [&]() -> float {
                    float mx[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t mword = mw[q];
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const float a0 = ((mword >> i) & 1u) ? __uint_as_float(sv[q][i]) : -INFINITY;
                            const float a1 = ((mword >> (i + 1)) & 1u) ? __uint_as_float(sv[q][i + 1]) : -INFINITY;
                            mx[(i >> 1) & 7] = fmax3(mx[(i >> 1) & 7], a0, a1);
                        }
                    }
                    return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
                };
                auto chunk_sum = [&]() -> float {
                    float sm[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) f2_unpack(sm2[i], sm[2 * i], sm[2 * i + 1]);
                    return ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
                };
                // The group's first chunk of an item takes the row maximum first and computes P against
                // it (a row may see no key of its block in a chunk: it keeps max -inf, P 0).  Later chunks
                // make one pass against the running reference maximum; while a row's sum stays at or
                // below RESCALE_SUM_LIMIT no P of it can overflow anything.  Otherwise (or for a row that
                // had seen no key yet) the chunk is redone from the registers: exact maximum, O rescaled,
                // P recomputed against it.
                float alpha = 1.0f;
                float sum;
                bool big = false;
                bool exact = !mine_any;
                for (;;) {
                    if (exact) {
                        const float mxs = max_pass();
                        if (!mine_any) {
                            m_ref = mxs;
                        } else {
                            const bool grow = big && mxs > m_ref;
                            const float m_new = grow ? mxs : m_ref;
                            alpha = grow ? ex2_approx(m_ref - m_new) : 1.0f;
                            m_ref = m_new;
                            rescale_o(alpha);   // O_w is quiet: the first exp pass waited for the previous PV
                        }
                    }
                    if (!exp_pass(-m_ref)) {
                        ok = false;
                        break;
                    }
                    sum = chunk_sum();
                    if (exact) break;
                    big = !(sum <= RESCALE_SUM_LIMIT);
                    if (!__any_sync(0xffffffffu, big)) break;
                    exact = true;
                }
                if (!ok) break;
                l = l * alpha + sum;
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ctl.p_full[w]));
                mine_any = true;
                ++n;
            }
            if (!ok) break;
            // ---- epilogue: wait for this group's last PV, swap (m, l), merge
            if (mine_any && !wait_warp(smem_u32(&ctl.p_free[w]), (n & 1) ^ 1, abort_flag, wlim)) break;
            if (!wait_warp(smem_u32(&ctl.mrg_empty), (item_seq & 1) ^ 1, abort_flag, wlim)) break;
            ctl.mrg_m[w][row] = m_ref;
            ctl.mrg_l[w][row] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl.mrg_full));
            if (!wait_warp(smem_u32(&ctl.mrg_full), item_seq & 1, abort_flag, wlim)) break;
            const float m0 = ctl.mrg_m[0][row], m1 = ctl.mrg_m[1][row];
            const float l0 = ctl.mrg_l[0][row], l1 = ctl.mrg_l[1][row];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl.mrg_empty));
            const float mm = fmaxf(m0, m1);
            // a group with no chunk in this item has l = 0 and m = -inf: weight 0
            const float a0 = l0 > 0.f ? ex2_approx(m0 - mm) : 0.f;
            const float a1 = l1 > 0.f ? ex2_approx(m1 - mm) : 0.f;
            // Which group holds which half of an item's chunks follows the CTA's chunk count, so the
            // merge is written symmetric in the two groups (products rounded separately, one add;
            // no contraction into an fma): the output bits do not depend on the schedule.
            const float inv = 1.0f / __fadd_rn(__fmul_rn(l0, a0), __fmul_rn(l1, a1));
            const float f0 = a0 * inv, f1 = a1 * inv;
            const bool use0 = __any_sync(0xffffffffu, l0 > 0.f), use1 = __any_sync(0xffffffffu, l1 > 0.f);
            tc_fence_after();
            const bool in_tile = GRP ? row < min(a.G, g.nb - qb) * bs : row < bs;   // rows of real query blocks
            __nv_bfloat16* orow;
            bool store;
            if (a.raster) {
                // the inverse reorder fused in: tile row -> raster token (b, n, h), padding rows dropped
                int tf_, ty_, tx_;
                const bool real = in_tile && token_of_pos(g, static_cast<long long>(qb) * bs + row, tf_, ty_, tx_);
                const long long b_ = bh / g.H, h_ = bh - b_ * g.H;
                const long long n_ = real ? (static_cast<long long>(tf_) * g.Hs + ty_) * g.Ws + tx_ : 0;
                orow = a.o + ((b_ * g.N + n_) * g.H + h_) * D;
                store = real;
            } else {
                orow = a.o + ((static_cast<long long>(bh) * g.Npad) + static_cast<long long>(qb) * bs + row) * D;
                store = in_tile;
            }
            // this group writes output columns [w*D/2, w*D/2 + D/2)
#pragma unroll 1
            for (int q = 0; q < D / 64; ++q) {
                const uint32_t col = static_cast<uint32_t>(w * (D / 2) + q * 32);
                float r[32], r1[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = r1[i] = 0.f;
                if (use0) {
                    uint32_t o0[32];
                    tmem_ld32(trow + O_COL + col, o0);
                    tmem_wait_ld();
                    if (l0 > 0.f) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __fmul_rn(__uint_as_float(o0[i]), f0);
                    }
                }
                if (use1) {
                    uint32_t o1[32];
                    tmem_ld32(trow + O_COL + 128u + col, o1);
                    tmem_wait_ld();
                    if (l1 > 0.f) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r1[i] = __fmul_rn(__uint_as_float(o1[i]), f1);
                    }
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __fadd_rn(r[i], r1[i]);
                if (store) {
#pragma unroll
                    for (int v8 = 0; v8 < 4; ++v8) {
                        uint4 wq;
                        wq.x = pack_bf16x2(r[v8 * 8 + 0], r[v8 * 8 + 1]);
                        wq.y = pack_bf16x2(r[v8 * 8 + 2], r[v8 * 8 + 3]);
                        wq.z = pack_bf16x2(r[v8 * 8 + 4], r[v8 * 8 + 5]);
                        wq.w = pack_bf16x2(r[v8 * 8 + 6], r[v8 * 8 + 7]);
                        *reinterpret_cast<uint4*>(orow + col + v8 * 8) = wq;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl.o_free));
            c_seq += nc;
            ++item_seq;
        }
    } else {
        regs_dec<RegSplit<GRP>::LOW>();
        if (warp == 0) {
            // =========================== K producer: items, Q tile, K blocks, masks
            // Column col = q*32 + lane of a chunk is token `off` of slot `slot`;
            // its frame / row / col offsets inside the tile never change.
            int c_slot[4], c_of[4], c_oy[4], c_ox[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int col = q * 32 + lane;
                c_slot[q] = col / bs;
                const int off = col - c_slot[q] * bs;
                c_ox[q] = off % g.tw;
                c_oy[q] = (off / g.tw) % g.th;
                c_of[q] = off / (g.tw * g.th);
            }
            int item_seq = 0;
            uint32_t c_seq = 0;      // K chunks loaded
            uint32_t q_fills = 0;    // Q tiles loaded
            bool ok = true;
            while (ok) {
                const int slot = item_seq & 1;
                if (!wait_warp(smem_u32(&ctl.item_empty[slot]), ((item_seq >> 1) & 1) ^ 1, abort_flag, wlim)) break;
                int t = 0;
                if (lane == 0) t = atomicAdd(a.counter, 1);
                t = __shfl_sync(0xffffffffu, t, 0);
                if (t >= a.total_items) {
                    if (lane == 0) {
                        ctl.item[slot][3] = 0;
                        mbar_arrive(smem_u32(&ctl.item_full[slot]));
                    }
                    break;
                }
                const int G = GRP ? a.G : 1;
                const int units = GRP ? a.ngroups : g.nb;
                const int hs = t / units;
                const int r = t - hs * units;
                const int bh = __ldg(a.head_order + hs);
                const int u = __ldg(a.item_order + static_cast<long long>(bh) * units + r);
                const int qb = u * G;                     // first query block of the tile
                const int nq = min(G, g.nb - qb);         // query blocks in the tile
                int cnt = GRP ? __ldg(a.gcnt + static_cast<long long>(bh) * a.ngroups + u)
                              : __ldg(a.kv_cnt + static_cast<long long>(bh) * g.nb + qb);
                if (cnt < 1 || cnt > g.nb) {
                    if (lane == 0) record_status(FVATTN_ERR_BOUNDS);
                    cnt = cnt < 1 ? 1 : g.nb;
                }
                if (lane == 0) {
                    ctl.item[slot][0] = bh;
                    ctl.item[slot][1] = qb;
                    ctl.item[slot][2] = cnt;
                    ctl.item[slot][3] = 1;
                    mbar_arrive(smem_u32(&ctl.item_full[slot]));
                }
                if (!wait_warp(smem_u32(&ctl.q_empty), (item_seq & 1) ^ 1, abort_flag, wlim)) break;
                const int row_base = bh * static_cast<int>(g.Npad);
                ++q_fills;
                if (lane == 0) {
                    mbar_arrive_expect_tx(smem_u32(&ctl.q_full), static_cast<uint32_t>(nq * bs * D * 2));
                    for (int tq = 0; tq < (GRP ? nq : 1); ++tq)
#pragma unroll
                        for (int h = 0; h < D / 64; ++h)
                            tma_load_2d(sQ + h * 16384u + static_cast<uint32_t>(tq * bs) * 128u, &tmQ, h * 64,
                                        row_base + (qb + tq) * bs, smem_u32(&ctl.q_full));
                }
                const int32_t* list = a.kv_idx + (static_cast<long long>(bh) * g.nb + qb) * g.nb;
                const uint32_t* ul = GRP ? a.ulist + (static_cast<long long>(bh) * a.ngroups + u) * g.nb : nullptr;
                const int nc = (cnt + bpc - 1) / bpc;
                // chunk cl's blocks (lane s < nblk: slot s), membership bits and real extents, one chunk
                // ahead (the extent load is in flight while the current chunk is handled)
                int j_next = 0;
                uint32_t m_next = 1u;
                int n_next = min(bpc, cnt);
                if (GRP) {
                    j_next = union_slot(ul, 0, bpc, n_next, lane, g.nb, m_next);
                } else {
                    j_next = chunk_block(list, 0, bpc, n_next, lane, g.nb);
                }
                int e_next = lane < n_next ? __ldg(a.ext + j_next) : 0;
                for (int cl = 0; cl < nc; ++cl, ++c_seq) {
                    const int stage = c_seq % KS;
                    const int nblk = n_next;
                    const int j = j_next;
                    const uint32_t mem = m_next;
                    const int ext = e_next;
                    if (cl + 1 < nc) {
                        n_next = min(bpc, cnt - (cl + 1) * bpc);
                        if (GRP) {
                            j_next = union_slot(ul, cl + 1, bpc, n_next, lane, g.nb, m_next);
                        } else {
                            j_next = chunk_block(list, cl + 1, bpc, n_next, lane, g.nb);
                        }
                        e_next = lane < n_next ? __ldg(a.ext + j_next) : 0;
                    }
                    if (!wait_warp(smem_u32(&ctl.k_empty[stage]), ((c_seq / KS) & 1) ^ 1, abort_flag, wlim)) {
                        ok = false;
                        break;
                    }
                    if (GRP) {
                        // per query block t of the tile: key column real and its block in t's list.
                        // Real-token bits once per 32-column word; a word lies in one slot when
                        // bs >= 32, so its membership bits are warp-uniform there.
                        uint32_t pad[4], mq[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int e = __shfl_sync(0xffffffffu, ext, c_slot[q]);
                            mq[q] = __shfl_sync(0xffffffffu, mem, c_slot[q]);
                            pad[q] = __ballot_sync(0xffffffffu, (c_of[q] < (e & 255)) && (c_oy[q] < ((e >> 8) & 255)) &&
                                                                    (c_ox[q] < (e >> 16)));
                        }
                        for (int tq = 0; tq < G; ++tq) {
                            uint32_t words[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                words[q] = bs >= 32 ? (((mq[q] >> tq) & 1u) ? pad[q] : 0u)
                                                    : (pad[q] & __ballot_sync(0xffffffffu, (mq[q] >> tq) & 1u));
                            if (lane == 0) {
#pragma unroll
                                for (int q = 0; q < 4; ++q) ctl.mask[stage][tq][q] = words[q];
                            }
                        }
                    } else {
                        (void)mem;
                        uint32_t words[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int e = __shfl_sync(0xffffffffu, ext, c_slot[q]);
                            const bool valid = (c_of[q] < (e & 255)) && (c_oy[q] < ((e >> 8) & 255)) && (c_ox[q] < (e >> 16));
                            words[q] = __ballot_sync(0xffffffffu, valid);
                        }
                        if (lane == 0) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) ctl.mask[stage][0][q] = words[q];
                        }
                    }
                    const uint32_t bar = smem_u32(&ctl.k_full[stage]);
                    if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nblk * bs * D * 2));
                    __syncwarp();
                    if (lane < nblk) {
                        const uint32_t kb = sK + stage * L::KV_BYTES + lane * bs * 128u;
#pragma unroll
                        for (int h = 0; h < D / 64; ++h) tma_load_2d(kb + h * 16384u, &tmK, h * 64, row_base + j * bs, bar);
                    }
                }
                ++item_seq;
            }
            // On the way out (also after an abort): wait for this warp's own loads in flight, the last
            // fill of every stage, so no copy into shared memory outlives the CTA.
            if (lane == 0) {
                if (q_fills > 0) wait_bar_drain(smem_u32(&ctl.q_full), (q_fills - 1) & 1, wlim);
                for (int st = 0; st < KS; ++st) {
                    const uint32_t fills = c_seq > static_cast<uint32_t>(st) ? (c_seq - st + KS - 1) / KS : 0u;
                    if (fills > 0) wait_bar_drain(smem_u32(&ctl.k_full[st]), (fills - 1) & 1, wlim);
                }
            }
            __syncwarp();
        } else if (warp == 2) {
            // =========================== V producer
            int item_seq = 0;
            uint32_t c_seq = 0;      // V chunks loaded
            // fault injection: this warp leaves at once, loading and arriving nothing, so the PV issuer's
            // wait for V must run out
            bool ok = (a.hooks & FVATTN_HOOK_SKIP_V_LOADS) == 0;
            while (ok) {
                const int slot = item_seq & 1;
                if (!wait_warp(smem_u32(&ctl.item_full[slot]), (item_seq >> 1) & 1, abort_flag, wlim)) break;
                const int bh = ctl.item[slot][0];
                const int qb = ctl.item[slot][1];
                const int cnt = ctl.item[slot][2];
                const int valid = ctl.item[slot][3];
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ctl.item_empty[slot]));
                if (!valid) break;
                const int row_base = bh * static_cast<int>(g.Npad);
                const int G = GRP ? a.G : 1;
                const int32_t* list = a.kv_idx + (static_cast<long long>(bh) * g.nb + qb) * g.nb;
                const uint32_t* ul = GRP ? a.ulist + (static_cast<long long>(bh) * a.ngroups + qb / G) * g.nb : nullptr;
                const int nc = (cnt + bpc - 1) / bpc;
                uint32_t m_unused = 0u;
                int n_next = min(bpc, cnt);
                int j_next = GRP ? union_slot(ul, 0, bpc, n_next, lane, g.nb, m_unused)
                                 : chunk_block(list, 0, bpc, n_next, lane, g.nb);
                for (int cl = 0; cl < nc; ++cl, ++c_seq) {
                    const int stage = c_seq % V_STAGES;
                    const int nblk = n_next;
                    const int j = j_next;
                    if (cl + 1 < nc) {
                        n_next = min(bpc, cnt - (cl + 1) * bpc);
                        j_next = GRP ? union_slot(ul, cl + 1, bpc, n_next, lane, g.nb, m_unused)
                                     : chunk_block(list, cl + 1, bpc, n_next, lane, g.nb);
                    }
                    if (!wait_warp(smem_u32(&ctl.v_empty[stage]), ((c_seq / V_STAGES) & 1) ^ 1, abort_flag, wlim)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = smem_u32(&ctl.v_full[stage]);
                    if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nblk * bs * D * 2));
                    __syncwarp();
                    if (lane < nblk) {
                        const uint32_t vb = sV + stage * L::KV_BYTES + lane * bs * 128u;
#pragma unroll
                        for (int h = 0; h < D / 64; ++h) tma_load_2d(vb + h * 16384u, &tmV, h * 64, row_base + j * bs, bar);
                    }
                }
                ++item_seq;
            }
            if (lane == 0) {
                for (int st = 0; st < V_STAGES; ++st) {
                    const uint32_t fills =
                        c_seq > static_cast<uint32_t>(st) ? (c_seq - st + V_STAGES - 1) / V_STAGES : 0u;
                    if (fills > 0) wait_bar_drain(smem_u32(&ctl.v_full[st]), (fills - 1) & 1, wlim);
                }
            }
            __syncwarp();
        } else if (warp == 1 || warp == 3) {
            // =========================== tensor-core issuers (one lane each)
            // Chunk c of the CTA's stream goes to softmax group w = c & 1 (S_w,
            // P_w, O_w).  Warp 1 issues S_w = Q K^T for every chunk, warp 3
            // issues O_w += P_w V.  Two issuing threads keep the tensor pipe fed:
            // while one waits on its barriers (a memory operation by the issuing
            // thread stalls until its own MMAs drain) the other's MMAs run.
            if (lane == 0) {
                const bool qk_role = warp == 1;
                constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
                constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
                int item_seq = 0;
                uint32_t c_seq = 0;
                uint32_t n0 = 0u, n1 = 0u;   // chunks handled per group
                unsigned long long blocks = 0;
                bool ok = true;
                while (ok) {
                    const int slot = item_seq & 1;
                    if (!wait_bar(smem_u32(&ctl.item_full[slot]), (item_seq >> 1) & 1, abort_flag, wlim)) break;
                    const int valid = ctl.item[slot][3];
                    const int cnt = ctl.item[slot][2];
                    mbar_arrive(smem_u32(&ctl.item_empty[slot]));
                    if (!valid) break;
                    const int nc = (cnt + bpc - 1) / bpc;
                    if (qk_role) {
                        blocks += static_cast<unsigned long long>(cnt);
                        if (!wait_bar(smem_u32(&ctl.q_full), item_seq & 1, abort_flag, wlim)) break;
                    } else {
                        // the item's first PV waits until the previous item's
                        // epilogue has read both accumulators
                        if (!wait_bar(smem_u32(&ctl.o_free), (item_seq & 1) ^ 1, abort_flag, wlim)) break;
                    }
                    for (int cl = 0; cl < nc; ++cl) {
                        const uint32_t c = c_seq + cl;
                        const int w = c & 1;
                        const uint32_t n = w ? n1 : n0;
                        if (qk_role) {
                            const int stage = c % KS;
                            if (!wait_bar2(smem_u32(&ctl.k_full[stage]), (c / KS) & 1, smem_u32(&ctl.s_free[w]),
                                           (n & 1) ^ 1, abort_flag, wlim)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t kb = sK + stage * L::KV_BYTES;
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                                const uint64_t ad = sw128_desc(sQ + off, 16u, 1024u);
                                const uint64_t bd = sw128_desc(kb + off, 16u, 1024u);
                                mma_bf16_ss(tmem + static_cast<uint32_t>(w) * 128u, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
                            }
                            mma_commit(smem_u32(&ctl.s_full[w]));
                            mma_commit(smem_u32(&ctl.k_empty[stage]));
                            if (cl == nc - 1) mma_commit(smem_u32(&ctl.q_empty));
                        } else {
                            const int stage = c % V_STAGES;
                            if (!wait_bar2(smem_u32(&ctl.p_full[w]), n & 1, smem_u32(&ctl.v_full[stage]),
                                           (c / V_STAGES) & 1, abort_flag, wlim)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t vb = sV + stage * L::KV_BYTES;
                            const uint32_t pb = sP + w * L::P_BYTES;
                            const uint32_t od = tmem + O_COL + static_cast<uint32_t>(w) * 128u;
                            const bool first = cl < 2;   // group w's first chunk of the item
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint64_t ad = sw128_desc(pb + (kk >> 2) * 16384u + (kk & 3) * 32u, 16u, 1024u);
                                const uint64_t bd = sw128_desc(vb + kk * 2048u, 16384u, 1024u);
                                mma_bf16_ss(od, ad, bd, IDESC_PV, (first && kk == 0) ? 0u : 1u);
                            }
                            mma_commit(smem_u32(&ctl.v_empty[stage]));
                            mma_commit(smem_u32(&ctl.p_free[w]));
                        }
                        if (w) ++n1; else ++n0;
                    }
                    if (!ok) break;
                    c_seq += nc;
                    ++item_seq;
                }
                if (qk_role) ctl.blocks_done = blocks;
                // every MMA this thread issued has completed (and made its commits) before the TMEM release
                mma_commit(smem_u32(&ctl.drain[qk_role ? 0 : 1]));
                wait_bar_drain(smem_u32(&ctl.drain[qk_role ? 0 : 1]), 0, wlim);
            }
            __syncwarp();
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
    if (threadIdx.x == 0 && a.sm_stats) {
        const unsigned long long t_end = global_timer_ns();
        a.sm_stats[blockIdx.x] = t_end - t_start;
        a.sm_stats[gridDim.x + blockIdx.x] = ctl.blocks_done;
    }
}

// ------------------------------------------------------------------ work list

// One warp per (b*h, query group) when G = 128 / bs > 1: the union of the
// group's G kv lists in ascending block order, each entry the block id with
// its membership bits (bit t: the block is in query block t's list) above
// bit 24, and the union's size, which is the number of kv blocks the group's
// tile walks.  Order and repeats inside a list do not matter.
__global__ void __launch_bounds__(256) group_union_kernel(Geo g, int G, int ngroups, int nwords,
                                                          const int32_t* __restrict__ kv_idx,
                                                          const int32_t* __restrict__ kv_cnt,
                                                          uint32_t* __restrict__ ulist, int32_t* __restrict__ gcnt) {
    extern __shared__ uint32_t gb_smem[];   // [8 warps][G * nwords] membership bitmaps
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long unit = static_cast<long long>(blockIdx.x) * 8 + warp;
    if (unit >= static_cast<long long>(g.B) * g.H * ngroups) return;
    const int nb = g.nb;
    const long long bh = unit / ngroups;
    const int grp = static_cast<int>(unit - bh * ngroups);
    uint32_t* bits = gb_smem + warp * G * nwords;
    for (int i = lane; i < G * nwords; i += 32) bits[i] = 0u;
    __syncwarp();
    for (int t = 0; t < G; ++t) {
        const int qb = grp * G + t;
        if (qb >= nb) break;
        int cnt = kv_cnt[bh * nb + qb];
        if (cnt < 1 || cnt > nb) {
            if (lane == 0) record_status(FVATTN_ERR_BOUNDS);
            cnt = cnt < 1 ? 1 : nb;
        }
        const int32_t* list = kv_idx + (bh * nb + qb) * nb;
        for (int e = lane; e < cnt; e += 32) {
            int j = list[e];
            if (j < 0 || j >= nb) {
                record_status(FVATTN_ERR_BOUNDS);
                j = 0;
            }
            atomicOr(&bits[t * nwords + (j >> 5)], 1u << (j & 31));
        }
    }
    __syncwarp();
    // lane l takes word 32r + l of round r; an exclusive scan of the words' union counts places them
    uint32_t* dst = ulist + unit * nb;
    int base = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
        const int wd = w0 + lane;
        uint32_t un = 0u;
        if (wd < nwords)
            for (int t = 0; t < G; ++t) un |= bits[t * nwords + wd];
        const int c = __popc(un);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int k = base + incl - c;
        for (uint32_t r = un; r != 0u; r &= r - 1u) {
            const int b = __ffs(static_cast<int>(r)) - 1;
            uint32_t mem = 0u;
            for (int t = 0; t < G; ++t) mem |= ((bits[t * nwords + wd] >> b) & 1u) << t;
            dst[k++] = static_cast<uint32_t>(wd * 32 + b) | (mem << 24);
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) gcnt[unit] = base;
}

// One CTA per (b, h): order the head's `units` work units (query blocks, or
// query groups when G > 1) by cost (kv blocks walked), longest first (ties by
// lower index), and record the head's total cost.
__global__ void __launch_bounds__(256) worklist_head_kernel(Geo g, int units, const int32_t* __restrict__ cost_in,
                                                            int32_t* __restrict__ item_order,
                                                            long long* __restrict__ head_cost) {
    extern __shared__ int wl_hist[];   // [nb + 2]
    const int nb = g.nb;
    const long long bh = blockIdx.x;
    const int32_t* cnt = cost_in + bh * units;
    for (int i = threadIdx.x; i < nb + 2; i += blockDim.x) wl_hist[i] = 0;
    __syncthreads();
    long long part = 0;
    for (int i = threadIdx.x; i < units; i += blockDim.x) {
        int c = cnt[i];
        c = c < 1 ? 1 : (c > nb ? nb : c);
        atomicAdd(&wl_hist[c], 1);
        part += c;
    }
    // block reduction of the cost
    __shared__ long long red[8];
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long tot = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
        head_cost[bh] = tot;
        // descending exclusive scan: start[c] = #units with a larger cost
        int run = 0;
        for (int c = nb; c >= 1; --c) {
            int h = wl_hist[c];
            wl_hist[c] = run;
            run += h;
        }
        // stable placement in ascending unit order
        for (int i = 0; i < units; ++i) {
            int c = cnt[i];
            c = c < 1 ? 1 : (c > nb ? nb : c);
            item_order[bh * units + wl_hist[c]++] = i;
        }
    }
}

// Single CTA: heads by total cost, heaviest first (ties by lower index);
// resets the item counter; writes every block's real extent.
__global__ void __launch_bounds__(256) worklist_heads_kernel(Geo g, int BH, const long long* __restrict__ head_cost,
                                                             int32_t* __restrict__ head_order, int* counter,
                                                             int32_t* __restrict__ ext) {
    for (int b = threadIdx.x; b < g.nb; b += blockDim.x) ext[b] = block_extent(g, b);
    for (int h = threadIdx.x; h < BH; h += blockDim.x) {
        const long long ch = head_cost[h];
        int rank = 0;
        for (int o = 0; o < BH; ++o) {
            const long long co = head_cost[o];
            rank += (co > ch) || (co == ch && o < h);
        }
        head_order[rank] = h;
    }
    if (threadIdx.x == 0) *counter = 0;
}

// ------------------------------------------------------------------ host side

// 2-D view [rows, D] of a tiled tensor, boxes of bs rows x 64 columns,
// 128-byte swizzle (the tcgen05 K-major / MN-major SW128 operand layout).
static bool make_tmap(CUtensorMap* m, const void* base, long long rows, int D, int bs) {
    return make_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, static_cast<unsigned long long>(rows),
                        static_cast<unsigned long long>(D), 64u, static_cast<unsigned>(bs));
}

// Workspace: work list (item order, head cost and order, counter), block
// extents and, when G = 128 / bs > 1, the query groups' union lists and sizes.
struct WsLayout {
    size_t item_order, head_cost, head_order, counter, ext, ulist, gcnt, total;
    int G, ngroups, nwords;
};

static size_t al256(size_t x) { return (x + 255) / 256 * 256; }

static WsLayout ws_layout(const fvattn_geom& g) {
    WsLayout w;
    size_t BH = static_cast<size_t>(g.B) * g.H;
    w.G = g.bs > 0 && g.bs < 128 ? 128 / g.bs : 1;
    w.ngroups = (g.nb + w.G - 1) / w.G;
    w.nwords = (g.nb + 31) / 32;
    w.item_order = 0;
    w.head_cost = al256(sizeof(int32_t) * BH * g.nb);
    w.head_order = w.head_cost + al256(sizeof(long long) * BH);
    w.counter = w.head_order + al256(sizeof(int32_t) * BH);
    w.ext = w.counter + 256;
    w.ulist = w.ext + al256(sizeof(int32_t) * g.nb);
    w.gcnt = w.ulist;
    w.total = w.ulist;
    if (w.G > 1) {
        w.gcnt = w.ulist + al256(sizeof(uint32_t) * BH * w.ngroups * g.nb);
        w.total = w.gcnt + al256(sizeof(int32_t) * BH * w.ngroups);
    }
    return w;
}

// Fault-injection settings of fvattn_test_hook (0: normal operation).
static std::atomic<unsigned long long> g_hook_wait_limit_ns{0};
static std::atomic<int> g_hook_flags{0};

static int cached_num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int D, bool GRP>
static int launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& args,
                       int grid, cudaStream_t s) {
    using L = Smem<D>;
    if (cudaFuncSetAttribute(sparse_attn_kernel<D, GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(L::ALLOC)) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    // The warpgroups' register shares (setmaxnreg) must fit in what a CTA is
    // launched with, or the raising warpgroups would wait for ever.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, sparse_attn_kernel<D, GRP>) != cudaSuccess) return FVATTN_ERR_CUDA;
    if (static_cast<long long>(fa.numRegs) * ATT_THREADS < 128ll * RegSplit<GRP>::LOW + 256ll * RegSplit<GRP>::HIGH)
        return FVATTN_ERR_UNSUPPORTED;
    sparse_attn_kernel<D, GRP><<<grid, ATT_THREADS, L::ALLOC, s>>>(tq, tk, tv, args);
    FV_CHECK_LAUNCH();
    return FVATTN_OK;
}

}  // namespace fv

using namespace fv;

extern "C" size_t fvattn_attn_workspace_size(const fvattn_geom* gp) {
    if (!gp) return 0;
    return ws_layout(*gp).total;
}

extern "C" int fvattn_num_sms(void) { return cached_num_sms(); }

extern "C" int fvattn_test_hook(unsigned long long wait_limit_ns, int flags) {
    if ((flags & ~FVATTN_HOOK_SKIP_V_LOADS) != 0) return FVATTN_ERR_INVALID;
    g_hook_wait_limit_ns.store(wait_limit_ns);
    g_hook_flags.store(flags);
    return FVATTN_OK;
}

static int attn_impl(const fvattn_geom* gp, const void* q_t, const void* k_t, const void* v_t, const int32_t* kv_idx,
                     const int32_t* kv_cnt, float scale, void* o_t, int raster, unsigned long long* sm_stats,
                     void* workspace, size_t ws_bytes, fvattn_stream_t stream) {
    if (!gp || !q_t || !k_t || !v_t || !kv_idx || !kv_cnt || !o_t || !workspace) return FVATTN_ERR_INVALID;
    if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(v_t) || !aligned16(o_t) || !aligned16(kv_idx) ||
        !aligned16(kv_cnt) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return FVATTN_ERR_INVALID;
    if (!isfinite(scale) || !(scale > 0.f)) return FVATTN_ERR_INVALID;
    if (gp->D != 64 && gp->D != 128) return FVATTN_ERR_UNSUPPORTED;
    if (gp->bs != 16 && gp->bs != 32 && gp->bs != 64 && gp->bs != 128) return FVATTN_ERR_UNSUPPORTED;
    if (gp->nb <= 0 || gp->nb > 2560) return FVATTN_ERR_UNSUPPORTED;
    const WsLayout wl = ws_layout(*gp);
    if (ws_bytes < wl.total) return FVATTN_ERR_INVALID;
    const long long rows = static_cast<long long>(gp->B) * gp->H * gp->Npad;
    if (rows >= (1ll << 31)) return FVATTN_ERR_UNSUPPORTED;
    Geo g = to_geo(*gp);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    int32_t* item_order = reinterpret_cast<int32_t*>(ws + wl.item_order);
    long long* head_cost = reinterpret_cast<long long*>(ws + wl.head_cost);
    int32_t* head_order = reinterpret_cast<int32_t*>(ws + wl.head_order);
    int* counter = reinterpret_cast<int*>(ws + wl.counter);
    uint32_t* ulist = wl.G > 1 ? reinterpret_cast<uint32_t*>(ws + wl.ulist) : nullptr;
    int32_t* gcnt = wl.G > 1 ? reinterpret_cast<int32_t*>(ws + wl.gcnt) : nullptr;
    const int BH = g.B * g.H;
    const int units = wl.G > 1 ? wl.ngroups : g.nb;

    if (wl.G > 1) {
        const long long warps = static_cast<long long>(BH) * wl.ngroups;
        group_union_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, sizeof(uint32_t) * 8 * wl.G * wl.nwords, s>>>(
            g, wl.G, wl.ngroups, wl.nwords, kv_idx, kv_cnt, ulist, gcnt);
        FV_CHECK_LAUNCH();
    }
    worklist_head_kernel<<<BH, 256, sizeof(int) * (g.nb + 2), s>>>(g, units, wl.G > 1 ? gcnt : kv_cnt, item_order,
                                                                   head_cost);
    FV_CHECK_LAUNCH();
    int32_t* ext = reinterpret_cast<int32_t*>(ws + wl.ext);
    worklist_heads_kernel<<<1, 256, 0, s>>>(g, BH, head_cost, head_order, counter, ext);
    FV_CHECK_LAUNCH();

    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, q_t, rows, g.D, g.bs) || !make_tmap(&tk, k_t, rows, g.D, g.bs) ||
        !make_tmap(&tv, v_t, rows, g.D, g.bs))
        return FVATTN_ERR_CUDA;
    AttnArgs args;
    args.g = g;
    args.kv_idx = kv_idx;
    args.kv_cnt = kv_cnt;
    args.head_order = head_order;
    args.item_order = item_order;
    args.counter = counter;
    args.o = static_cast<__nv_bfloat16*>(o_t);
    args.raster = raster;
    args.sm_stats = sm_stats;
    args.scale_log2 = scale * 1.4426950408889634f;
    args.G = wl.G;
    args.ngroups = wl.ngroups;
    args.ulist = ulist;
    args.gcnt = gcnt;
    args.ext = ext;
    args.total_items = BH * units;
    const unsigned long long hook_limit = g_hook_wait_limit_ns.load();
    args.wait_limit_ns = hook_limit ? hook_limit : WAIT_LIMIT_NS;
    args.hooks = g_hook_flags.load();
    int nsm = cached_num_sms();
    if (nsm <= 0) return FVATTN_ERR_CUDA;
    const int grid = nsm;
    if (wl.G > 1)
        return g.D == 128 ? launch_attn<128, true>(tq, tk, tv, args, grid, s)
                          : launch_attn<64, true>(tq, tk, tv, args, grid, s);
    return g.D == 128 ? launch_attn<128, false>(tq, tk, tv, args, grid, s)
                      : launch_attn<64, false>(tq, tk, tv, args, grid, s);
}

extern "C" int fvattn_sparse_attn(const fvattn_geom* gp, const void* q_t, const void* k_t, const void* v_t,
                                  const int32_t* kv_idx, const int32_t* kv_cnt, float scale, void* o_t,
                                  unsigned long long* sm_stats, void* workspace, size_t ws_bytes,
                                  fvattn_stream_t stream) {
    return attn_impl(gp, q_t, k_t, v_t, kv_idx, kv_cnt, scale, o_t, 0, sm_stats, workspace, ws_bytes, stream);
}

extern "C" int fvattn_sparse_attn_raster(const fvattn_geom* gp, const void* q_t, const void* k_t, const void* v_t,
                                         const int32_t* kv_idx, const int32_t* kv_cnt, float scale, void* o,
                                         unsigned long long* sm_stats, void* workspace, size_t ws_bytes,
                                         fvattn_stream_t stream) {
    return attn_impl(gp, q_t, k_t, v_t, kv_idx, kv_cnt, scale, o, 1, sm_stats, workspace, ws_bytes, stream);
}

int fv::take_status_attn() { return fv::take_tu_status(); }
