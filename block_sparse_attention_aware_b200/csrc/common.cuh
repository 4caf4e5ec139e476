// Shared definitions of the CUDA path: geometry passed to kernels, the
// device status word, and the tile <-> raster index maps.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "fvattn.h"

namespace fv {

// Kernel-side copy of the geometry (plain ints, passed by value).
struct Geo {
    int B, H, D, F, Hs, Ws, tf, th, tw;
    int nbf, nby, nbx, bs, nb;
    long long N, Npad;
    const int32_t* order;   // block order table (2*nb), or null for raster tile order
};

inline Geo to_geo(const fvattn_geom& g) {
    Geo k;
    k.B = g.B; k.H = g.H; k.D = g.D; k.F = g.F; k.Hs = g.Hs; k.Ws = g.Ws;
    k.tf = g.tf; k.th = g.th; k.tw = g.tw;
    k.nbf = g.nbf; k.nby = g.nby; k.nbx = g.nbx; k.bs = g.bs; k.nb = g.nb;
    k.N = g.N; k.Npad = g.Npad;
    k.order = g.order;
    return k;
}

// Device status word of this translation unit: FVATTN_OK or the first error
// one of its kernels recorded.  Every .cu file is compiled as a whole
// program (no relocatable device code: ptxas then honours the per-warpgroup
// register budgets of setmaxnreg), so each owns one word;
// fvattn_get_status reads and clears them all through the take_status_*
// functions below.
static __device__ int g_tu_status = 0;

__device__ __forceinline__ void record_status(int code) {
    atomicCAS(&g_tu_status, 0, code);
}

// Host side: read this translation unit's status word on the current device
// and clear it; FVATTN_ERR_CUDA if the copy fails.
static inline int take_tu_status() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tu_status, sizeof(int)) != cudaSuccess) return FVATTN_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_tu_status, &zero, sizeof(int)) != cudaSuccess) return FVATTN_ERR_CUDA;
    return v;
}

// The status words of the files whose kernels record errors.
int take_status_route();
int take_status_attn();

// Raster tile index of a block, and block of a raster tile (identities in
// raster tile order).
__device__ __forceinline__ int tile_of_block(const Geo& g, int block) {
    return g.order ? __ldg(g.order + block) : block;
}

__device__ __forceinline__ long long block_of_tile(const Geo& g, long long tile) {
    return g.order ? static_cast<long long>(__ldg(g.order + g.nb + tile)) : tile;
}

// Raster token (f, y, x) of tile-layout position `pos` of a head, and
// whether it is a real token.
__device__ __forceinline__ bool token_of_pos(const Geo& g, long long pos, int& f, int& y, int& x) {
    int block = static_cast<int>(pos / g.bs);
    int off = static_cast<int>(pos - static_cast<long long>(block) * g.bs);
    block = tile_of_block(g, block);
    int bx = block % g.nbx;
    int rest = block / g.nbx;
    int by = rest % g.nby;
    int bf = rest / g.nby;
    int ox = off % g.tw;
    int r2 = off / g.tw;
    int oy = r2 % g.th;
    int of = r2 / g.th;
    f = bf * g.tf + of;
    y = by * g.th + oy;
    x = bx * g.tw + ox;
    return f < g.F && y < g.Hs && x < g.Ws;
}

}  // namespace fv

#define FV_CHECK_LAUNCH()                                      \
    do {                                                       \
        cudaError_t e_ = cudaGetLastError();                   \
        if (e_ != cudaSuccess) return FVATTN_ERR_CUDA;         \
    } while (0)
