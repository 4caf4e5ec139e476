// Video-aware block organisation and its inverse (FVAttn pages,
// paperlayer.ai summary, section 3 "FVAttn Design": "Sparse-routing
// frontend" groups spatially adjacent tokens into blocks; "Pipeline" ends by
// restoring the original layout).
//
// Both kernels are HBM-bound bit copies.  A warp owns 32 consecutive
// destination rows: each lane decodes one row's source address once, then
// the warp streams the 32 rows as 16-byte vectors, two (D = 128) or four
// (D = 64) rows per instruction, so every access is a full 256/128-byte
// contiguous run.  All loads of a warp's 32 rows are issued before the
// stores.  The reorder numbers its warps head-fastest (warp = (b, 32-row
// chunk of a head's tiled rows, h)), so the warps running at one time read
// every head of the same raster tokens, one contiguous H * D run per token,
// rather than one row every H * D elements.
#include "common.cuh"

namespace fv {

template <int VPR>  // 16-byte vectors per row = D / 8
__global__ void __launch_bounds__(256) reorder_kernel(Geo g, const uint4* __restrict__ x,
                                                      uint4* __restrict__ xt, long long warps) {
    const int lane = threadIdx.x & 31;
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (warp >= warps) return;
    const long long chunks = (g.Npad + 31) / 32;
    const int h = static_cast<int>(warp % g.H);
    const long long bc = warp / g.H;
    const long long pos0 = (bc % chunks) * 32;                   // first tiled row of the chunk in its head
    const int b = static_cast<int>(bc / chunks);
    const long long row0 = (static_cast<long long>(b) * g.H + h) * g.Npad + pos0;
    const long long nrows = g.Npad - pos0 < 32 ? g.Npad - pos0 : 32;
    // destination row -> source row (raster), or -1 for padding
    long long src_row = -1;
    if (lane < nrows) {
        int f, y, xx;
        if (token_of_pos(g, pos0 + lane, f, y, xx)) {
            long long n = (static_cast<long long>(f) * g.Hs + y) * g.Ws + xx;
            src_row = (static_cast<long long>(b) * g.N + n) * g.H + h;
        }
    }
    constexpr int ITER = VPR;  // 32 rows * VPR vectors / 32 lanes
    uint4 v[ITER];
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        int q = it * 32 + lane;
        int rl = q / VPR, vec = q % VPR;
        long long s = __shfl_sync(0xffffffffu, src_row, rl);
        v[it] = make_uint4(0, 0, 0, 0);
        if (s >= 0) v[it] = __ldg(x + s * VPR + vec);
    }
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        int q = it * 32 + lane;
        int rl = q / VPR, vec = q % VPR;
        if (rl < nrows) xt[(row0 + rl) * VPR + vec] = v[it];
    }
}

template <int VPR>
__global__ void __launch_bounds__(256) inverse_reorder_kernel(Geo g, const uint4* __restrict__ xt,
                                                              uint4* __restrict__ x, long long rows) {
    const int lane = threadIdx.x & 31;
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long row0 = warp * 32;
    if (row0 >= rows) return;
    long long src_row = 0;
    const long long r = row0 + lane;
    if (r < rows) {
        // destination raster row r = (b*N + n)*H + h
        long long bn = r / g.H;
        int h = static_cast<int>(r - bn * g.H);
        long long b = bn / g.N;
        long long n = bn - b * g.N;
        int xx = static_cast<int>(n % g.Ws);
        long long fy = n / g.Ws;
        int y = static_cast<int>(fy % g.Hs);
        int f = static_cast<int>(fy / g.Hs);
        long long block = block_of_tile(g, (static_cast<long long>(f / g.tf) * g.nby + y / g.th) * g.nbx + xx / g.tw);
        long long off = (static_cast<long long>(f % g.tf) * g.th + y % g.th) * g.tw + xx % g.tw;
        src_row = (b * g.H + h) * g.Npad + block * g.bs + off;
    }
    constexpr int ITER = VPR;
    uint4 v[ITER];
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        int q = it * 32 + lane;
        int rl = q / VPR, vec = q % VPR;
        long long s = __shfl_sync(0xffffffffu, src_row, rl);
        if (row0 + rl < rows) v[it] = __ldg(xt + s * VPR + vec);
    }
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        int q = it * 32 + lane;
        int rl = q / VPR, vec = q % VPR;
        if (row0 + rl < rows) x[(row0 + rl) * VPR + vec] = v[it];
    }
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace fv

using namespace fv;

extern "C" int fvattn_reorder(const fvattn_geom* gp, const void* x, void* x_tiled,
                              fvattn_stream_t stream) {
    if (!gp || !x || !x_tiled || !aligned16(x) || !aligned16(x_tiled)) return FVATTN_ERR_INVALID;
    if (gp->bs <= 0 || gp->nb <= 0) return FVATTN_ERR_INVALID;
    Geo g = to_geo(*gp);
    long long warps = static_cast<long long>(g.B) * g.H * ((g.Npad + 31) / 32);
    long long blocks = (warps * 32 + 255) / 256;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (g.D == 128)
        reorder_kernel<16><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            g, static_cast<const uint4*>(x), static_cast<uint4*>(x_tiled), warps);
    else if (g.D == 64)
        reorder_kernel<8><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            g, static_cast<const uint4*>(x), static_cast<uint4*>(x_tiled), warps);
    else
        return FVATTN_ERR_UNSUPPORTED;
    FV_CHECK_LAUNCH();
    return FVATTN_OK;
}

extern "C" int fvattn_inverse_reorder(const fvattn_geom* gp, const void* o_tiled, void* o,
                                      fvattn_stream_t stream) {
    if (!gp || !o || !o_tiled || !aligned16(o) || !aligned16(o_tiled)) return FVATTN_ERR_INVALID;
    if (gp->bs <= 0 || gp->nb <= 0) return FVATTN_ERR_INVALID;
    Geo g = to_geo(*gp);
    long long rows = static_cast<long long>(g.B) * g.N * g.H;
    long long warps = (rows + 31) / 32;
    long long blocks = (warps * 32 + 255) / 256;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (g.D == 128)
        inverse_reorder_kernel<16><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            g, static_cast<const uint4*>(o_tiled), static_cast<uint4*>(o), rows);
    else if (g.D == 64)
        inverse_reorder_kernel<8><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            g, static_cast<const uint4*>(o_tiled), static_cast<uint4*>(o), rows);
    else
        return FVATTN_ERR_UNSUPPORTED;
    FV_CHECK_LAUNCH();
    return FVATTN_OK;
}
