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
//   select_kernel  One warp per (b, h, query block) row, the row's logits in
//                  registers.  Probability masses e_j = exp(L_j - max L) are
//                  48-bit fixed point, so every partial sum is an exact integer
//                  independent of summation order.  The first prefix (logit
//                  descending, index ascending) whose mass reaches p * total
//                  (Top-p) and the min(k, nb)-th entry (Top-k floor) are found
//                  by linear bucketing of the logit range into 256 buckets with
//                  a mass/count histogram, refined inside the boundary bucket
//                  until at most 32 candidates remain, which one warp sorts
//                  (bitonic) and scans.  Equal logits go by ascending index.
//                  The kept indices are written in ascending order with ballots.
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
constexpr int SEL_MAX_LEVELS = 4;

// Order key of (logit, index): ascending key = logit descending, then index
// ascending.  -0 is folded into +0 so that equal logits get equal keys.
__device__ __forceinline__ unsigned long long order_key(float v, int j) {
    const uint32_t b = __float_as_uint(v + 0.0f);
    const uint32_t asc = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return (static_cast<unsigned long long>(~asc) << 32) | static_cast<uint32_t>(j);
}

// Probability mass exp(l - lmax) in (0, 1] as 48-bit fixed point; with at
// most 2560 entries every sum stays below 2^60.
__device__ __forceinline__ unsigned long long fixed_mass(float l, float lmax) {
    return static_cast<unsigned long long>(__expf(l - lmax) * 281474976710656.0f);
}

struct SelSmem {
    unsigned int cnt[256];
    unsigned long long mass[256];
    unsigned long long ckey[32];
    unsigned long long cmass[32];
};

// Refinement levels of the boundary search: the candidates are the entries
// whose level-t bucket equals bsel[t] for every level t < n.
struct Levels {
    float hi[SEL_MAX_LEVELS];
    float scl[SEL_MAX_LEVELS];
    int bsel[SEL_MAX_LEVELS];
    int n;
};

// Monotone bucket of a logit inside [lo, hi]: larger logits, lower buckets.
__device__ __forceinline__ int lin_bucket(float v, float hi, float scl) {
    const int b = static_cast<int>((hi - v) * scl);
    return b < 255 ? b : 255;
}

__device__ __forceinline__ bool in_levels(float v, const Levels& lv) {
    bool in = true;
#pragma unroll
    for (int t = 0; t < SEL_MAX_LEVELS; ++t)
        if (t < lv.n) in = in && lin_bucket(v, lv.hi[t], lv.scl[t]) == lv.bsel[t];
    return in;
}

// Boundary of the weighted prefix: the first entry, in (logit desc, index
// asc) order, at which the running weight (fixed-point mass, or 1 per entry
// when use_mass is false) reaches `target`.  Returns its order key; *rank is
// its 1-based position.  If the target is never reached, returns ~0ull.
// Slow path, taken only when a boundary bucket holds more than 32 entries:
// the same search, refined level by level, re-reading the row from memory.
__device__ __noinline__ unsigned long long find_boundary(const float* __restrict__ Lr, int nb, float lmax, float lmin,
                                                         bool use_mass, double target, SelSmem& sm, int* rank) {
    const int lane = threadIdx.x & 31;
    Levels lv;
    lv.n = 0;
    double before = 0.0;        // weight of all entries ordered before the candidate set
    int before_c = 0;
    float hi = lmax, lo = lmin;
    unsigned int ccount = static_cast<unsigned int>(nb);
#pragma unroll 1
    for (int level = 0; level <= SEL_MAX_LEVELS; ++level) {
        if (hi == lo) {
            // every candidate carries the same logit: take them by index
            const unsigned long long each = use_mass ? fixed_mass(hi, lmax) : 1ull;
            const double need = target - before;
            long long t = each ? static_cast<long long>(ceil(need / static_cast<double>(each))) : 1;
            if (t < 1) t = 1;
            if (t > static_cast<long long>(ccount)) t = ccount;
            int seen = 0;
            unsigned long long key = ~0ull;
            for (int j0 = 0; j0 < nb; j0 += 32) {
                const int j = j0 + lane;
                const float x = j < nb ? Lr[j] + 0.0f : 0.f;
                const bool c = j < nb && x == hi && in_levels(x, lv);
                const unsigned int bal = __ballot_sync(0xffffffffu, c);
                const int pos = seen + __popc(bal & ((1u << lane) - 1u));
                if (c && pos + 1 == t) key = order_key(x, j);
                seen += __popc(bal);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) key = min(key, __shfl_xor_sync(0xffffffffu, key, o));
            *rank = before_c + static_cast<int>(t);
            return key;
        }
        if (ccount <= 32u || level == SEL_MAX_LEVELS) {
            // at most 32 candidates: gather, sort by order key, scan
            int seen = 0;
            for (int j0 = 0; j0 < nb; j0 += 32) {
                const int j = j0 + lane;
                const float x = j < nb ? Lr[j] + 0.0f : 0.f;
                const bool c = j < nb && in_levels(x, lv);
                const unsigned int bal = __ballot_sync(0xffffffffu, c);
                if (c) {
                    const int pos = seen + __popc(bal & ((1u << lane) - 1u));
                    if (pos < 32) {
                        sm.ckey[pos] = order_key(x, j);
                        sm.cmass[pos] = use_mass ? fixed_mass(x, lmax) : 1ull;
                    }
                }
                seen += __popc(bal);
            }
            if (seen > 32) return ~0ull;   // cannot happen for finite logits
            __syncwarp();
            unsigned long long key = lane < seen ? sm.ckey[lane] : ~0ull;
            unsigned long long w = lane < seen ? sm.cmass[lane] : 0ull;
            __syncwarp();
            // bitonic sort of (key, w) ascending by key across the warp
#pragma unroll
            for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
                for (int stride = size >> 1; stride > 0; stride >>= 1) {
                    const unsigned long long ok = __shfl_xor_sync(0xffffffffu, key, stride);
                    const unsigned long long ow = __shfl_xor_sync(0xffffffffu, w, stride);
                    const bool ascending = (lane & size) == 0;
                    const bool lower = (lane & stride) == 0;
                    const bool swap = (ascending == lower) ? (ok < key) : (ok > key);
                    if (swap) {
                        key = ok;
                        w = ow;
                    }
                }
            }
            // inclusive prefix of the weights in sorted order
            unsigned long long pre = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long t = __shfl_up_sync(0xffffffffu, pre, o);
                if (lane >= o) pre += t;
            }
            const bool hit = lane < seen && before + static_cast<double>(pre) >= target;
            const unsigned int bal = __ballot_sync(0xffffffffu, hit);
            if (bal == 0u) return ~0ull;
            const int src = __ffs(bal) - 1;
            *rank = before_c + src + 1;
            return __shfl_sync(0xffffffffu, key, src);
        }
        // histogram of the candidates over 256 linear buckets of [lo, hi]
        const float scl = 256.0f / (hi - lo);
        for (int b = lane; b < 256; b += 32) {
            sm.cnt[b] = 0u;
            sm.mass[b] = 0ull;
        }
        __syncwarp();
        for (int j = lane; j < nb; j += 32) {
            const float x = Lr[j] + 0.0f;
            if (in_levels(x, lv)) {
                const int b = lin_bucket(x, hi, scl);
                atomicAdd(&sm.cnt[b], 1u);
                if (use_mass) atomicAdd(&sm.mass[b], fixed_mass(x, lmax));
            }
        }
        __syncwarp();
        // first bucket at which the running weight reaches the target
        unsigned long long wb[8];
        unsigned int cb[8];
        unsigned long long wsum = 0;
        unsigned int csum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            cb[e] = sm.cnt[lane * 8 + e];
            wb[e] = use_mass ? sm.mass[lane * 8 + e] : static_cast<unsigned long long>(cb[e]);
            wsum += wb[e];
            csum += cb[e];
        }
        unsigned long long wex = wsum;
        unsigned int cex = csum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long tw = __shfl_up_sync(0xffffffffu, wex, o);
            const unsigned int tc = __shfl_up_sync(0xffffffffu, cex, o);
            if (lane >= o) {
                wex += tw;
                cex += tc;
            }
        }
        wex -= wsum;
        cex -= csum;
        int found = -1;
        double run = before + static_cast<double>(wex);
        int runc = before_c + static_cast<int>(cex);
        double run_at = 0.0;
        int runc_at = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (found < 0 && cb[e] > 0u && run + static_cast<double>(wb[e]) >= target) {
                found = lane * 8 + e;
                run_at = run;
                runc_at = runc;
            }
            run += static_cast<double>(wb[e]);
            runc += static_cast<int>(cb[e]);
        }
        const unsigned int bal = __ballot_sync(0xffffffffu, found >= 0);
        if (bal == 0u) return ~0ull;
        const int src = __ffs(bal) - 1;
        const int bsel = __shfl_sync(0xffffffffu, found, src);
        before = __shfl_sync(0xffffffffu, run_at, src);
        before_c = __shfl_sync(0xffffffffu, runc_at, src);
        ccount = sm.cnt[bsel];
        __syncwarp();
#pragma unroll
        for (int t = 0; t < SEL_MAX_LEVELS; ++t)
            if (t == lv.n) {
                lv.hi[t] = hi;
                lv.scl[t] = scl;
                lv.bsel[t] = bsel;
            }
        ++lv.n;
        // the candidate range for the next level
        float nhi = -INFINITY, nlo = INFINITY;
        for (int j = lane; j < nb; j += 32) {
            const float x = Lr[j] + 0.0f;
            if (in_levels(x, lv)) {
                nhi = fmaxf(nhi, x);
                nlo = fminf(nlo, x);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            nhi = fmaxf(nhi, __shfl_xor_sync(0xffffffffu, nhi, o));
            nlo = fminf(nlo, __shfl_xor_sync(0xffffffffu, nlo, o));
        }
        hi = nhi;
        lo = nlo;
    }
    return ~0ull;
}

// Gather the (at most 32) entries flagged by `pick`, sort them by order key
// and return the first at which before + running weight reaches `target`
// (key and 1-based rank within the sorted set).  ~0ull if never reached.
template <int NPL, class Pick>
__device__ __forceinline__ unsigned long long sort_scan_pick(const float (&v)[NPL], int nb, float lmax, bool use_mass,
                                                             double before, double target, SelSmem& sm, Pick pick,
                                                             int* rank) {
    const int lane = threadIdx.x & 31;
    int seen = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int j = lane + 32 * i;
        const bool c = j < nb && pick(i);
        const unsigned int bal = __ballot_sync(0xffffffffu, c);
        if (c) {
            const int pos = seen + __popc(bal & ((1u << lane) - 1u));
            sm.ckey[pos] = order_key(v[i], j);
            sm.cmass[pos] = use_mass ? fixed_mass(v[i], lmax) : 1ull;
        }
        seen += __popc(bal);
    }
    __syncwarp();
    unsigned long long key = lane < seen ? sm.ckey[lane] : ~0ull;
    unsigned long long w = lane < seen ? sm.cmass[lane] : 0ull;
    __syncwarp();
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const unsigned long long ok = __shfl_xor_sync(0xffffffffu, key, stride);
            const unsigned long long ow = __shfl_xor_sync(0xffffffffu, w, stride);
            const bool ascending = (lane & size) == 0;
            const bool lower = (lane & stride) == 0;
            const bool swap = (ascending == lower) ? (ok < key) : (ok > key);
            if (swap) {
                key = ok;
                w = ow;
            }
        }
    }
    unsigned long long pre = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long t = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += t;
    }
    const unsigned int bal = __ballot_sync(0xffffffffu, lane < seen && before + static_cast<double>(pre) >= target);
    if (bal == 0u) return ~0ull;
    const int src = __ffs(bal) - 1;
    *rank = src + 1;
    return __shfl_sync(0xffffffffu, key, src);
}

// Shared first level: every entry's bucket among 256 linear buckets of
// [lmin, lmax] (packed four per word), per-bucket counts and fixed-point
// masses.  Then for each target (mass reaching p * total; count reaching
// min(k, nb)) the boundary bucket is resolved directly when it holds at most
// 32 entries; larger boundary buckets fall back to find_boundary.
template <int NPL>
__global__ void __launch_bounds__(32 * SEL_WARPS) select_kernel(int nb, long long rows, const float* __restrict__ L,
                                                                double p, int kfloor, int32_t* __restrict__ kv_idx,
                                                                int32_t* __restrict__ kv_cnt) {
    __shared__ SelSmem sel[SEL_WARPS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * SEL_WARPS + warp;
    if (row >= rows) return;
    SelSmem& sm = sel[warp];
    const float* Lr = L + row * nb;
    float v[NPL];
    float lmax = -INFINITY, lmin = INFINITY;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int j = lane + 32 * i;
        v[i] = j < nb ? Lr[j] + 0.0f : 0.f;
        if (j < nb) {
            lmax = fmaxf(lmax, v[i]);
            lmin = fminf(lmin, v[i]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        lmin = fminf(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
    }
    const int kf = min(kfloor, nb);
    unsigned long long thr = ~0ull;   // keep every entry whose order key is <= thr
    if (p < 1.0) {
        const float scl = lmax > lmin ? 256.0f / (lmax - lmin) : 0.f;
        for (int b = lane; b < 256; b += 32) {
            sm.cnt[b] = 0u;
            sm.mass[b] = 0ull;
        }
        __syncwarp();
        uint32_t bk[(NPL + 3) / 4];
#pragma unroll
        for (int q = 0; q < (NPL + 3) / 4; ++q) bk[q] = 0u;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            if (lane + 32 * i < nb) {
                const int b = lin_bucket(v[i], lmax, scl);
                bk[i >> 2] |= static_cast<uint32_t>(b) << (8 * (i & 3));
                atomicAdd(&sm.cnt[b], 1u);
                atomicAdd(&sm.mass[b], fixed_mass(v[i], lmax));
            }
        }
        __syncwarp();
        // per-lane bucket chunks (8 buckets a lane) and exclusive prefixes
        unsigned long long wb[8];
        unsigned int cb[8];
        unsigned long long wsum = 0;
        unsigned int csum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            cb[e] = sm.cnt[lane * 8 + e];
            wb[e] = sm.mass[lane * 8 + e];
            wsum += wb[e];
            csum += cb[e];
        }
        unsigned long long wex = wsum, tot = wsum;
        unsigned int cex = csum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long tw = __shfl_up_sync(0xffffffffu, wex, o);
            const unsigned int tc = __shfl_up_sync(0xffffffffu, cex, o);
            if (lane >= o) {
                wex += tw;
                cex += tc;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        wex -= wsum;
        cex -= csum;
        const double target = p * static_cast<double>(tot);
        // boundary bucket of the mass target and of the count target
        int fm = -1, fk = -1;
        double bm = 0.0;
        int bcm = 0, bck = 0;
        {
            double run = static_cast<double>(wex);
            unsigned int runc = cex;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (fm < 0 && cb[e] > 0u && run + static_cast<double>(wb[e]) >= target) {
                    fm = lane * 8 + e;
                    bm = run;
                    bcm = static_cast<int>(runc);
                }
                if (fk < 0 && cb[e] > 0u && static_cast<int>(runc + cb[e]) >= kf) {
                    fk = lane * 8 + e;
                    bck = static_cast<int>(runc);
                }
                run += static_cast<double>(wb[e]);
                runc += cb[e];
            }
        }
        const unsigned int balm = __ballot_sync(0xffffffffu, fm >= 0);
        const unsigned int balk = __ballot_sync(0xffffffffu, fk >= 0);
        if (balm != 0u) {
            const int sm_ = __ffs(balm) - 1;
            const int b_m = __shfl_sync(0xffffffffu, fm, sm_);
            const double before_m = __shfl_sync(0xffffffffu, bm, sm_);
            const int before_cm = __shfl_sync(0xffffffffu, bcm, sm_);
            const unsigned int n_m = sm.cnt[b_m];
            int rank = 0;
            unsigned long long kp;
            if (n_m <= 32u) {
                kp = sort_scan_pick<NPL>(v, nb, lmax, true, before_m, target, sm,
                                         [&](int i) { return static_cast<int>((bk[i >> 2] >> (8 * (i & 3))) & 255u) == b_m; },
                                         &rank);
                rank += before_cm;
            } else {
                kp = find_boundary(Lr, nb, lmax, lmin, true, target, sm, &rank);
            }
            if (kp != ~0ull) {
                thr = kp;
                if (rank < kf && balk != 0u) {
                    const int sk = __ffs(balk) - 1;
                    const int b_k = __shfl_sync(0xffffffffu, fk, sk);
                    const int before_ck = __shfl_sync(0xffffffffu, bck, sk);
                    const unsigned int n_k = sm.cnt[b_k];
                    int rk = 0;
                    if (n_k <= 32u) {
                        thr = sort_scan_pick<NPL>(v, nb, lmax, false, static_cast<double>(before_ck), static_cast<double>(kf),
                                                  sm,
                                                  [&](int i) { return static_cast<int>((bk[i >> 2] >> (8 * (i & 3))) & 255u) == b_k; },
                                                  &rk);
                    } else {
                        thr = find_boundary(Lr, nb, lmax, lmin, false, static_cast<double>(kf), sm, &rk);
                    }
                }
            }
        }
    }
    // emit the kept indices in ascending order
    int32_t* out = kv_idx + row * nb;
    int written = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int j = lane + 32 * i;
        const bool keep = j < nb && order_key(v[i], j) <= thr;
        const unsigned int bal = __ballot_sync(0xffffffffu, keep);
        if (keep) out[written + __popc(bal & ((1u << lane) - 1u))] = j;
        written += __popc(bal);
    }
    if (lane == 0) kv_cnt[row] = written;
}

template <int NPL>
static int launch_select(long long rows, int nb, const float* L, double p, int kfloor, int32_t* kv_idx,
                         int32_t* kv_cnt, cudaStream_t s) {
    const long long blocks = (rows + SEL_WARPS - 1) / SEL_WARPS;
    select_kernel<NPL><<<static_cast<unsigned>(blocks), 32 * SEL_WARPS, 0, s>>>(nb, rows, L, p, kfloor, kv_idx,
                                                                              kv_cnt);
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
    if (g.nb <= 768) return launch_select<24>(rows, g.nb, L, p, k_floor, kv_idx, kv_cnt, s);
    if (g.nb <= 1536) return launch_select<48>(rows, g.nb, L, p, k_floor, kv_idx, kv_cnt, s);
    return launch_select<80>(rows, g.nb, L, p, k_floor, kv_idx, kv_cnt, s);
}
