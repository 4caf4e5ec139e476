// Sparse-routing frontend of FVAttn (paperlayer.ai summary, section 3
// "FVAttn Design", item "Sparse-routing frontend": Top-p CDF thresholding of
// each query block's similarity distribution plus a Top-k floor; section 2:
// Top-p keeps the smallest cumulative-importance set, the Top-k safety floor
// a minimum budget; dynamic masks come from the current attention features).
//
// Three kernels:
//   pool_kernel    HBM-bound.  One CTA per (tensor, b, h, block) sums the
//                  block's real rows with 16-byte loads, all issued before the
//                  first add (padding rows are never read), and writes the fp32
//                  mean.
//   score_kernel   L = scale * Qp Kp^T per (b, h): an fp32 register-tiled
//                  product, 64 x 64 logits per CTA, 4 x 4 per thread, operands
//                  staged in shared memory k-major.
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
#include "common.cuh"
#include "ptx.cuh"

namespace fv {

// ------------------------------------------------------------------ pooling

// One warp per (tensor, b, h, block); 8 warps per CTA.  A lane owns one
// 16-byte column slice (D/8 slices per row) of every (32 / (D/8))-th row, so
// one warp instruction reads 512 contiguous bytes; full tiles issue all their
// loads before the first add.
template <int D>
__global__ void __launch_bounds__(256, 3) pool_kernel(Geo g, const __nv_bfloat16* __restrict__ qt,
                                                   const __nv_bfloat16* __restrict__ kt,
                                                   float* __restrict__ qp, float* __restrict__ kp) {
    constexpr int VPR = D / 8;             // 16-byte vectors per row
    constexpr int RPI = 32 / VPR;          // rows per warp instruction
    constexpr int UNR = 8;                 // loads in flight per lane
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
    float* dst = (is_k ? kp : qp) + (bh * g.nb + blk) * D;
    const int vec = lane % VPR;
    const int r0 = lane / VPR;
    const int bx = blk % g.nbx, by = (blk / g.nbx) % g.nby, bf = blk / (g.nbx * g.nby);
    const int nf = min(g.tf, g.F - bf * g.tf);
    const int ny = min(g.th, g.Hs - by * g.th);
    const int nx = min(g.tw, g.Ws - bx * g.tw);
    const bool full = nf == g.tf && ny == g.th && nx == g.tw;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
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
        for (int i = 0; i < UNR; ++i) {
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u[i]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(p2[e]);
                acc[2 * e] += f.x;
                acc[2 * e + 1] += f.y;
            }
        }
    }
    // lanes with the same column slice hold partial sums of different rows
#pragma unroll
    for (int o = VPR; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (lane < VPR) {
        const float inv = 1.0f / static_cast<float>(nf * ny * nx);
        float4* d4 = reinterpret_cast<float4*>(dst + lane * 8);
        d4[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        d4[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    }
}

// ------------------------------------------------------------------ scores

constexpr int SC_TILE = 64;   // logits per CTA side
constexpr int SC_KC = 32;     // head-dim slice staged per step

// L[bh][i][j] = scale * <Qp[bh][i], Kp[bh][j]>; grid (tiles_j, tiles_i, B*H).
__global__ void __launch_bounds__(256) score_kernel(Geo g, const float* __restrict__ qp, const float* __restrict__ kp,
                                                    float scale, float* __restrict__ L) {
    __shared__ __align__(16) float As[SC_KC][SC_TILE + 4];
    __shared__ __align__(16) float Bs[SC_KC][SC_TILE + 4];
    const int nb = g.nb, D = g.D;
    const long long bh = blockIdx.z;
    const int i0 = blockIdx.y * SC_TILE, j0 = blockIdx.x * SC_TILE;
    const float* A = qp + bh * nb * D;
    const float* Bm = kp + bh * nb * D;
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    for (int k0 = 0; k0 < D; k0 += SC_KC) {
        // 64 rows x 32 floats of each operand: 512 float4, two per thread,
        // stored transposed (k-major)
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
            const int idx = tid + rep * 256;
            const int r = idx / (SC_KC / 4), c4 = idx % (SC_KC / 4);
            float4 va = make_float4(0.f, 0.f, 0.f, 0.f), vb = va;
            if (i0 + r < nb) va = __ldg(reinterpret_cast<const float4*>(A + static_cast<long long>(i0 + r) * D + k0) + c4);
            if (j0 + r < nb) vb = __ldg(reinterpret_cast<const float4*>(Bm + static_cast<long long>(j0 + r) * D + k0) + c4);
            As[c4 * 4 + 0][r] = va.x; As[c4 * 4 + 1][r] = va.y; As[c4 * 4 + 2][r] = va.z; As[c4 * 4 + 3][r] = va.w;
            Bs[c4 * 4 + 0][r] = vb.x; Bs[c4 * 4 + 1][r] = vb.y; Bs[c4 * 4 + 2][r] = vb.z; Bs[c4 * 4 + 3][r] = vb.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < SC_KC; ++k) {
            const float4 a = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
            const float4 b = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int i = i0 + ty * 4 + x;
        if (i >= nb) continue;
        float* row = L + (bh * nb + i) * nb;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int j = j0 + tx * 4 + y;
            if (j < nb) row[j] = acc[x][y] * scale;
        }
    }
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
__device__ unsigned long long sel_boundary(const float (&v)[NPL], const float (&e)[NPL], int nb, float lmax, float lmin,
                                           bool mass, int c_all, double target,
                                           unsigned long long* ck, int* rank) {
    const int lane = threadIdx.x & 31;
    uint32_t lo_k = fkey(lmin), hi_k = fkey(lmax) + 1u;
    unsigned long long s_hi = 0ull;
    int c_lo = c_all, c_hi = 0;
    (void)nb;
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

// One warp per (b, h, query block) row.  Kept set: every entry whose order key
// is at most that of the later of the Top-p crossing (first prefix whose mass
// reaches p * total) and the min(k, nb)-th entry.
template <int NPL, bool KEEP_E>
__global__ void __launch_bounds__(32 * SEL_WARPS, NPL <= 24 ? 3 : 1) select_kernel(int nb, long long rows, const float* __restrict__ L,
                                                                double p, int kfloor, int32_t* __restrict__ kv_idx,
                                                                int32_t* __restrict__ kv_cnt) {
    __shared__ unsigned long long cand_keys[SEL_WARPS][32];
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
        sel_eval<NPL, KEEP_E>(v, e, lmax, lmin, true, s_all, c_all);
        const double target = p * static_cast<double>(s_all);
        int rank = 0;
        thr = sel_boundary<NPL, KEEP_E>(v, e, nb, lmax, lmin, true, c_all, target, cand_keys[warp], &rank);
        if (rank < kf)
            thr = sel_boundary<NPL, KEEP_E>(v, e, nb, lmax, lmin, false, c_all, static_cast<double>(kf),
                                            cand_keys[warp], &rank);
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
static int launch_select(long long rows, int nb, const float* L, double p, int kfloor, int32_t* kv_idx,
                         int32_t* kv_cnt, cudaStream_t s) {
    const long long blocks = (rows + SEL_WARPS - 1) / SEL_WARPS;
    select_kernel<NPL, KEEP_E><<<static_cast<unsigned>(blocks), 32 * SEL_WARPS, 0, s>>>(nb, rows, L, p, kfloor,
                                                                                      kv_idx, kv_cnt);
    FV_CHECK_LAUNCH();
    return FVATTN_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct RouteWs {
    size_t qp, kp, logits, total;
};

static size_t al256(size_t x) { return (x + 255) / 256 * 256; }

static RouteWs route_ws(const fvattn_geom& g) {
    RouteWs w;
    const size_t BH = static_cast<size_t>(g.B) * g.H;
    const size_t pooled = al256(sizeof(float) * BH * g.nb * g.D);
    w.qp = 0;
    w.kp = pooled;
    w.logits = 2 * pooled;
    w.total = w.logits + al256(sizeof(float) * BH * g.nb * g.nb);
    return w;
}

}  // namespace fv

using namespace fv;

extern "C" size_t fvattn_route_workspace_size(const fvattn_geom* gp) {
    if (!gp) return 0;
    return route_ws(*gp).total;
}

extern "C" int fvattn_route(const fvattn_geom* gp, const void* q_tiled, const void* k_tiled, double p, int k_floor,
                            float scale, int32_t* kv_idx, int32_t* kv_cnt, float* q_pool, float* k_pool,
                            float* logits, void* workspace, size_t ws_bytes, fvattn_stream_t stream) {
    if (!gp || !q_tiled || !k_tiled || !kv_idx || !kv_cnt) return FVATTN_ERR_INVALID;
    if (!aligned16(q_tiled) || !aligned16(k_tiled) || !aligned16(kv_idx) || !aligned16(kv_cnt))
        return FVATTN_ERR_INVALID;
    if (!(p > 0.0 && p <= 1.0) || k_floor < 1 || !isfinite(scale)) return FVATTN_ERR_INVALID;
    if (gp->nb <= 0 || gp->nb > 2560) return FVATTN_ERR_UNSUPPORTED;
    if (gp->D != 64 && gp->D != 128) return FVATTN_ERR_UNSUPPORTED;
    const Geo g = to_geo(*gp);
    const RouteWs wl = route_ws(*gp);
    char* ws = static_cast<char*>(workspace);
    const bool need_ws = !q_pool || !k_pool || !logits;
    if (need_ws && (!workspace || ws_bytes < wl.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
        return FVATTN_ERR_INVALID;
    float* qp = q_pool ? q_pool : reinterpret_cast<float*>(ws + wl.qp);
    float* kp = k_pool ? k_pool : reinterpret_cast<float*>(ws + wl.kp);
    float* L = logits ? logits : reinterpret_cast<float*>(ws + wl.logits);
    if (!aligned16(qp) || !aligned16(kp) || !aligned16(L)) return FVATTN_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long units = 2ll * g.B * g.H * g.nb;
    const unsigned pblocks = static_cast<unsigned>((units + 7) / 8);
    if (g.D == 128)
        pool_kernel<128><<<pblocks, 256, 0, s>>>(g, static_cast<const __nv_bfloat16*>(q_tiled),
                                                 static_cast<const __nv_bfloat16*>(k_tiled), qp, kp);
    else
        pool_kernel<64><<<pblocks, 256, 0, s>>>(g, static_cast<const __nv_bfloat16*>(q_tiled),
                                                static_cast<const __nv_bfloat16*>(k_tiled), qp, kp);
    FV_CHECK_LAUNCH();
    const int tiles = (g.nb + SC_TILE - 1) / SC_TILE;
    score_kernel<<<dim3(tiles, tiles, g.B * g.H), 256, 0, s>>>(g, qp, kp, scale, L);
    FV_CHECK_LAUNCH();
    const long long rows = static_cast<long long>(g.B) * g.H * g.nb;
    if (g.nb <= 768) return launch_select<24, true>(rows, g.nb, L, p, k_floor, kv_idx, kv_cnt, s);
    if (g.nb <= 1536) return launch_select<48, true>(rows, g.nb, L, p, k_floor, kv_idx, kv_cnt, s);
    return launch_select<80, false>(rows, g.nb, L, p, k_floor, kv_idx, kv_cnt, s);
}
