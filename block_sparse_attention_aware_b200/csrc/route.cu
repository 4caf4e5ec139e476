// Sparse-routing frontend of FVAttn (paperlayer.ai summary, section 3
// "FVAttn Design", item "Sparse-routing frontend": Top-p CDF thresholding of
// each query block's similarity distribution plus a Top-k floor; section 2:
// Top-p keeps the smallest cumulative-importance set, the Top-k safety floor
// a minimum budget; dynamic masks come from the current attention features).
//
// Two kernels:
//   pool_kernel          HBM-bound.  One CTA per (tensor, b, h, block) sums the
//                        block's real rows with 16-byte loads (padding rows are
//                        never read) and writes the fp32 mean.
//   score_select_kernel  One CTA per (b, h, 32 query blocks).  Scores
//                        L = scale * Qp Kp^T for its 32 rows against every key
//                        block into shared memory (fp32 FMA, register-tiled),
//                        then one warp per row selects the kept set:
//                          - masses e_j = exp(L_j - max L) as 48-bit fixed
//                            point, so partial sums are exact integers and do
//                            not depend on summation order;
//                          - a most-significant-digit radix select over the
//                            order key (logit descending, index ascending)
//                            finds the first prefix whose mass reaches
//                            p * total (Top-p), and a second, count-based one
//                            the min(k, nb)-th entry (Top-k floor) when needed;
//                          - the kept indices are written in ascending order
//                            with ballots.
#include "common.cuh"
#include "ptx.cuh"

namespace fv {

// ------------------------------------------------------------------ pooling

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(Geo g, const __nv_bfloat16* __restrict__ qt,
                                                   const __nv_bfloat16* __restrict__ kt,
                                                   float* __restrict__ qp, float* __restrict__ kp) {
    constexpr int VPR = D / 8;            // 16-byte vectors per row
    constexpr int RG = 256 / VPR;         // rows handled per pass
    __shared__ float red[RG][D + 1];
    const int blk = blockIdx.x;
    const long long bh = blockIdx.y;
    const bool is_k = blockIdx.z != 0;
    const __nv_bfloat16* src = (is_k ? kt : qt) + (bh * g.Npad + static_cast<long long>(blk) * g.bs) * D;
    float* dst = (is_k ? kp : qp) + (bh * g.nb + blk) * D;

    const int vec = threadIdx.x % VPR;
    const int rg = threadIdx.x / VPR;
    // extents of this tile that hold real tokens
    const int bx = blk % g.nbx, by = (blk / g.nbx) % g.nby, bf = blk / (g.nbx * g.nby);
    const int nf = min(g.tf, g.F - bf * g.tf);
    const int ny = min(g.th, g.Hs - by * g.th);
    const int nx = min(g.tw, g.Ws - bx * g.tw);

    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int r = rg; r < g.bs; r += RG) {
        const int ox = r % g.tw, oy = (r / g.tw) % g.th, of = r / (g.tw * g.th);
        if (of >= nf || oy >= ny || ox >= nx) continue;
        uint4 u = __ldg(reinterpret_cast<const uint4*>(src + static_cast<long long>(r) * D) + vec);
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(p2[i]);
            acc[2 * i] += f.x;
            acc[2 * i + 1] += f.y;
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[rg][vec * 8 + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < D) {
        float s = 0.f;
        for (int i = 0; i < RG; ++i) s += red[i][threadIdx.x];
        dst[threadIdx.x] = s / static_cast<float>(nf * ny * nx);
    }
}

// ------------------------------------------------------------------ score + select

constexpr int SS_KCH = 64;       // key blocks per staged chunk
constexpr int SS_THREADS = 256;
constexpr int SS_WARPS = SS_THREADS / 32;

// Order key: ascending key = descending logit.  -0 is folded into +0 so that
// equal logits always get equal keys.
__device__ __forceinline__ uint32_t desc_key(float v) {
    uint32_t b = __float_as_uint(v + 0.0f);
    uint32_t asc = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ~asc;
}

__device__ __forceinline__ unsigned long long fixed_mass(float l, float lmax) {
    // e in (0, 1]; 2^48 * e <= 2^48, and nb <= 2560 keeps sums below 2^60.
    float e = __expf(l - lmax);
    return static_cast<unsigned long long>(e * 281474976710656.0f);
}

struct SelWarpSmem {
    unsigned int cnt[256];
    unsigned long long mass[256];
};

// Most-significant-digit radix select over the 32-bit order key.  Finds
// the key u* of the entry at which the running total (fixed-point mass or
// count, taken in key order) first reaches `target`, and how many entries
// with key exactly u* (equal logits, taken by ascending index) are needed.
// The caller passes the smallest and largest key of the row; bits above the
// highest bit in which they differ are shared by every entry and are fixed
// from the start.  If the target is never reached every entry is kept
// (u* = 0xFFFFFFFF, which no finite logit maps to).
__device__ __forceinline__ void radix_select(const float* __restrict__ L, int nb, float lmax, bool use_mass,
                             double target, uint32_t umin, uint32_t umax,
                             unsigned long long total, SelWarpSmem& sm, uint32_t& u_star,
                             int& take_ties, int& before_cnt) {
    const int lane = threadIdx.x & 31;
    const uint32_t diff = umin ^ umax;
    int hb = diff ? 31 - __clz(diff) : -1;            // highest undecided bit
    uint32_t pmask = (hb >= 31) ? 0u : (0xFFFFFFFFu << (hb + 1));
    uint32_t prefix = umin & pmask;
    double before = 0.0;
    int before_c = 0;
    unsigned int bucket_cnt = static_cast<unsigned int>(nb);
    unsigned long long bucket_w = use_mass ? total : static_cast<unsigned long long>(nb);
    while (hb >= 0) {
        const int width = hb + 1 < 8 ? hb + 1 : 8;
        const int shift = hb + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        for (int i = lane; i < 256; i += 32) {
            sm.cnt[i] = 0;
            sm.mass[i] = 0ull;
        }
        __syncwarp();
        for (int j = lane; j < nb; j += 32) {
            uint32_t u = desc_key(L[j]);
            if ((u & pmask) != prefix) continue;
            uint32_t dgt = (u >> shift) & dmask;
            atomicAdd(&sm.cnt[dgt], 1u);
            if (use_mass) atomicAdd(&sm.mass[dgt], fixed_mass(L[j], lmax));
        }
        __syncwarp();
        unsigned long long w[8];
        unsigned int c[8];
        unsigned long long wsum = 0;
        unsigned int csum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            c[i] = sm.cnt[lane * 8 + i];
            w[i] = use_mass ? sm.mass[lane * 8 + i] : static_cast<unsigned long long>(c[i]);
            wsum += w[i];
            csum += c[i];
        }
        unsigned long long wex = wsum;
        unsigned int cex = csum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            unsigned long long tw = __shfl_up_sync(0xffffffffu, wex, o);
            unsigned int tc = __shfl_up_sync(0xffffffffu, cex, o);
            if (lane >= o) { wex += tw; cex += tc; }
        }
        wex -= wsum;
        cex -= csum;
        int found = -1;
        double run = before + static_cast<double>(wex);
        int runc = before_c + static_cast<int>(cex);
        double run_at = 0.0;
        int runc_at = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (found < 0 && c[i] > 0 && run + static_cast<double>(w[i]) >= target) {
                found = lane * 8 + i;
                run_at = run;
                runc_at = runc;
            }
            run += static_cast<double>(w[i]);
            runc += static_cast<int>(c[i]);
        }
        const unsigned int ball = __ballot_sync(0xffffffffu, found >= 0);
        if (ball == 0u) {
            u_star = 0xFFFFFFFFu;
            take_ties = nb;
            before_cnt = 0;
            return;
        }
        const int src = __ffs(ball) - 1;
        const int dgt = __shfl_sync(0xffffffffu, found, src);
        before = __shfl_sync(0xffffffffu, run_at, src);
        before_c = __shfl_sync(0xffffffffu, runc_at, src);
        bucket_cnt = sm.cnt[dgt];
        bucket_w = use_mass ? sm.mass[dgt] : static_cast<unsigned long long>(bucket_cnt);
        __syncwarp();
        prefix |= static_cast<uint32_t>(dgt) << shift;
        pmask |= dmask << shift;
        hb = shift - 1;
        if (bucket_cnt == 1u && hb >= 0) {
            // the bucket's single entry fixes the remaining bits
            uint32_t u_found = 0u;
            for (int j = lane; j < nb; j += 32) {
                uint32_t u = desc_key(L[j]);
                if ((u & pmask) == prefix) u_found = u;
            }
            prefix = __reduce_or_sync(0xffffffffu, u_found);
            hb = -1;
        }
    }
    if (diff == 0u && !use_mass) bucket_w = static_cast<unsigned long long>(nb);
    // every entry with key == prefix has the same logit, hence the same weight
    const unsigned long long each = bucket_w / bucket_cnt;
    const double need = target - before;
    long long t = (each > 0ull) ? static_cast<long long>(ceil(need / static_cast<double>(each)))
                                : static_cast<long long>(bucket_cnt);
    if (t < 1) t = 1;
    if (t > static_cast<long long>(bucket_cnt)) t = bucket_cnt;
    u_star = prefix;
    take_ties = static_cast<int>(t);
    before_cnt = before_c;
}

// ROWS query blocks per CTA (32, or 16 when a row of logits is long).
template <int D, int ROWS>
__global__ void __launch_bounds__(SS_THREADS) score_select_kernel(
    Geo g, const float* __restrict__ qp, const float* __restrict__ kp, float scale, double p,
    int kfloor, int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt,
    float* __restrict__ logits_out) {
    extern __shared__ __align__(16) unsigned char ss_smem[];
    constexpr int DP = D + 4;  // padded row (floats), keeps 16-byte alignment
    const int nb = g.nb;
    const long long bh = blockIdx.y;
    constexpr int RPT = ROWS / 16;  // rows per thread
    const int row0 = blockIdx.x * ROWS;
    const int nrows = min(ROWS, nb - row0);
    float* Ls = reinterpret_cast<float*>(ss_smem);                     // [ROWS][nb]
    float* Qs = Ls + ROWS * nb;                                          // [ROWS][DP]
    float* Ks = Qs + ROWS * DP;                                          // [SS_KCH][DP]
    SelWarpSmem* sel = reinterpret_cast<SelWarpSmem*>(Qs);               // reuses Qs/Ks later

    const int tid = threadIdx.x;
    // stage the 32 query rows
    for (int i = tid; i < ROWS * (D / 4); i += SS_THREADS) {
        int r = i / (D / 4), c4 = i % (D / 4);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < nrows) v = __ldg(reinterpret_cast<const float4*>(qp + (bh * nb + row0 + r) * D) + c4);
        *reinterpret_cast<float4*>(Qs + r * DP + c4 * 4) = v;
    }
    const int ty = tid / 16;   // rows RPT*ty .. RPT*ty + RPT-1
    const int tx = tid % 16;   // keys tx + 16c
    for (int kc = 0; kc < nb; kc += SS_KCH) {
        const int nk = min(SS_KCH, nb - kc);
        __syncthreads();
        for (int i = tid; i < SS_KCH * (D / 4); i += SS_THREADS) {
            int r = i / (D / 4), c4 = i % (D / 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < nk) v = __ldg(reinterpret_cast<const float4*>(kp + (bh * nb + kc + r) * D) + c4);
            *reinterpret_cast<float4*>(Ks + r * DP + c4 * 4) = v;
        }
        __syncthreads();
        float acc[RPT][4];
#pragma unroll
        for (int a = 0; a < RPT; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
            float4 q[RPT];
#pragma unroll
            for (int a = 0; a < RPT; ++a)
                q[a] = *reinterpret_cast<const float4*>(Qs + (RPT * ty + a) * DP + d);
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                float4 k4 = *reinterpret_cast<const float4*>(Ks + (tx + 16 * b) * DP + d);
#pragma unroll
                for (int a = 0; a < RPT; ++a) {
                    acc[a][b] = fmaf(q[a].x, k4.x, acc[a][b]);
                    acc[a][b] = fmaf(q[a].y, k4.y, acc[a][b]);
                    acc[a][b] = fmaf(q[a].z, k4.z, acc[a][b]);
                    acc[a][b] = fmaf(q[a].w, k4.w, acc[a][b]);
                }
            }
        }
#pragma unroll
        for (int a = 0; a < RPT; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                int key = tx + 16 * b;
                if (key < nk) Ls[(RPT * ty + a) * nb + kc + key] = acc[a][b] * scale;
            }
    }
    __syncthreads();
    if (logits_out) {
        for (int i = tid; i < nrows * nb; i += SS_THREADS) {
            int r = i / nb, j = i % nb;
            logits_out[(bh * nb + row0 + r) * nb + j] = Ls[r * nb + j];
        }
    }
    // ---- selection, one warp per row
    const int warp = tid / 32, lane = tid % 32;
    SelWarpSmem& sm = sel[warp];
    const int kf = min(kfloor, nb);
    for (int r = warp; r < nrows; r += SS_WARPS) {
        const float* Lr = Ls + r * nb;
        const long long row = bh * nb + row0 + r;
        int32_t* out = kv_idx + row * nb;
        uint32_t u_star = 0xFFFFFFFFu;
        int take = nb, before = nb;
        if (p < 1.0 || kf < nb) {
            float lmax = -INFINITY;
            uint32_t umin = 0xFFFFFFFFu, umax = 0u;
            for (int j = lane; j < nb; j += 32) {
                float v = Lr[j];
                lmax = fmaxf(lmax, v);
                uint32_t u = desc_key(v);
                umin = min(umin, u);
                umax = max(umax, u);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
            umin = __reduce_min_sync(0xffffffffu, umin);
            umax = __reduce_max_sync(0xffffffffu, umax);
            int mp = nb;
            if (p < 1.0) {
                unsigned long long tot = 0;
                for (int j = lane; j < nb; j += 32) tot += fixed_mass(Lr[j], lmax);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
                const double target = p * static_cast<double>(tot);
                radix_select(Lr, nb, lmax, true, target, umin, umax, tot, sm, u_star, take, before);
                mp = (u_star == 0xFFFFFFFFu) ? nb : before + take;
            }
            if (mp < kf) {
                radix_select(Lr, nb, lmax, false, static_cast<double>(kf), umin, umax, 0ull, sm,
                             u_star, take, before);
            } else if (p >= 1.0) {
                u_star = 0xFFFFFFFFu;
            }
        }
        // emit ascending: keep u < u*, or u == u* among the first `take` ties
        int written = 0, ties_seen = 0;
        for (int j0 = 0; j0 < nb; j0 += 32) {
            int j = j0 + lane;
            bool in = j < nb;
            uint32_t u = in ? desc_key(Lr[j]) : 0xFFFFFFFFu;
            bool tie = in && (u == u_star);
            unsigned int tb = __ballot_sync(0xffffffffu, tie);
            int tie_rank = ties_seen + __popc(tb & ((1u << lane) - 1u));
            bool keep = in && ((u < u_star) || (tie && tie_rank < take));
            if (u_star == 0xFFFFFFFFu && in) keep = true;
            unsigned int kb = __ballot_sync(0xffffffffu, keep);
            if (keep) out[written + __popc(kb & ((1u << lane) - 1u))] = j;
            written += __popc(kb);
            ties_seen += __popc(tb);
        }
        if (lane == 0) kv_cnt[row] = written;
        __syncwarp();
    }
}

static size_t ss_smem_bytes(int nb, int D, int rows) {
    size_t ls = sizeof(float) * rows * static_cast<size_t>(nb);
    size_t qk = sizeof(float) * (rows + SS_KCH) * static_cast<size_t>(D + 4);
    size_t sel = sizeof(SelWarpSmem) * SS_WARPS;
    return ls + (qk > sel ? qk : sel);
}

template <int D, int ROWS>
static int launch_score_select(const Geo& g, const float* qp, const float* kp, float scale,
                               double p, int kfloor, int32_t* kv_idx, int32_t* kv_cnt,
                               float* logits, cudaStream_t s) {
    size_t smem = ss_smem_bytes(g.nb, D, ROWS);
    if (cudaFuncSetAttribute(score_select_kernel<D, ROWS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    dim3 grid((g.nb + ROWS - 1) / ROWS, g.B * g.H);
    score_select_kernel<D, ROWS><<<grid, SS_THREADS, smem, s>>>(g, qp, kp, scale, p, kfloor,
                                                                kv_idx, kv_cnt, logits);
    FV_CHECK_LAUNCH();
    return FVATTN_OK;
}

// Largest shared-memory footprint the score/select kernel may use.
constexpr size_t SS_SMEM_LIMIT = 220 * 1024;

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace fv

using namespace fv;

extern "C" size_t fvattn_route_workspace_size(const fvattn_geom* gp) {
    if (!gp) return 0;
    size_t pooled = sizeof(float) * static_cast<size_t>(gp->B) * gp->H * gp->nb * gp->D;
    return 2 * ((pooled + 255) / 256) * 256;
}

extern "C" int fvattn_route(const fvattn_geom* gp, const void* q_tiled, const void* k_tiled,
                            double p, int k_floor, float scale, int32_t* kv_idx, int32_t* kv_cnt,
                            float* q_pool, float* k_pool, float* logits, void* workspace,
                            size_t ws_bytes, fvattn_stream_t stream) {
    if (!gp || !q_tiled || !k_tiled || !kv_idx || !kv_cnt) return FVATTN_ERR_INVALID;
    if (!aligned16(q_tiled) || !aligned16(k_tiled) || !aligned16(kv_idx) || !aligned16(kv_cnt))
        return FVATTN_ERR_INVALID;
    if (!(p > 0.0 && p <= 1.0) || k_floor < 1 || !isfinite(scale)) return FVATTN_ERR_INVALID;
    if (gp->nb <= 0 || gp->nb > 2560) return FVATTN_ERR_UNSUPPORTED;
    if (gp->D != 64 && gp->D != 128) return FVATTN_ERR_UNSUPPORTED;
    Geo g = to_geo(*gp);
    size_t pooled = sizeof(float) * static_cast<size_t>(g.B) * g.H * g.nb * g.D;
    size_t pooled_al = (pooled + 255) / 256 * 256;
    float* qp = q_pool;
    float* kp = k_pool;
    if (!qp || !kp) {
        if (!workspace || ws_bytes < 2 * pooled_al ||
            (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return FVATTN_ERR_INVALID;
        if (!qp) qp = reinterpret_cast<float*>(workspace);
        if (!kp) kp = reinterpret_cast<float*>(static_cast<char*>(workspace) + pooled_al);
    }
    if (!aligned16(qp) || !aligned16(kp)) return FVATTN_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool rows32 = ss_smem_bytes(g.nb, g.D, 32) <= SS_SMEM_LIMIT;
    dim3 pg(g.nb, g.B * g.H, 2);
    int rc;
    if (g.D == 128) {
        pool_kernel<128><<<pg, 256, 0, s>>>(g, static_cast<const __nv_bfloat16*>(q_tiled),
                                            static_cast<const __nv_bfloat16*>(k_tiled), qp, kp);
        FV_CHECK_LAUNCH();
        rc = rows32 ? launch_score_select<128, 32>(g, qp, kp, scale, p, k_floor, kv_idx, kv_cnt, logits, s)
                    : launch_score_select<128, 16>(g, qp, kp, scale, p, k_floor, kv_idx, kv_cnt, logits, s);
    } else {
        pool_kernel<64><<<pg, 256, 0, s>>>(g, static_cast<const __nv_bfloat16*>(q_tiled),
                                           static_cast<const __nv_bfloat16*>(k_tiled), qp, kp);
        FV_CHECK_LAUNCH();
        rc = rows32 ? launch_score_select<64, 32>(g, qp, kp, scale, p, k_floor, kv_idx, kv_cnt, logits, s)
                    : launch_score_select<64, 16>(g, qp, kp, scale, p, k_floor, kv_idx, kv_cnt, logits, s);
    }
    return rc;
}
