// Geometry set-up and the device status word of the FVAttn C ABI.
#include "common.cuh"

using namespace fv;

static int ceil_div_i(int a, int b) { return (a + b - 1) / b; }

extern "C" int fvattn_geom_init(fvattn_geom* g) {
    if (!g) return FVATTN_ERR_INVALID;
    if (g->B < 1 || g->H < 1 || g->D < 1 || g->F < 1 || g->Hs < 1 || g->Ws < 1 || g->tf < 1 ||
        g->th < 1 || g->tw < 1)
        return FVATTN_ERR_INVALID;
    if (g->D != 64 && g->D != 128) return FVATTN_ERR_UNSUPPORTED;
    const long long bs = static_cast<long long>(g->tf) * g->th * g->tw;
    if (bs != 16 && bs != 32 && bs != 64 && bs != 128) return FVATTN_ERR_UNSUPPORTED;
    g->nbf = ceil_div_i(g->F, g->tf);
    g->nby = ceil_div_i(g->Hs, g->th);
    g->nbx = ceil_div_i(g->Ws, g->tw);
    g->Fp = g->nbf * g->tf;
    g->Hp = g->nby * g->th;
    g->Wp = g->nbx * g->tw;
    g->bs = static_cast<int>(bs);
    const long long nb = static_cast<long long>(g->nbf) * g->nby * g->nbx;
    if (nb > 2560) return FVATTN_ERR_UNSUPPORTED;
    g->nb = static_cast<int>(nb);
    g->N = static_cast<long long>(g->F) * g->Hs * g->Ws;
    g->Npad = nb * bs;
    g->order = nullptr;
    if (static_cast<long long>(g->B) * g->H * g->Npad >= (1ll << 31)) return FVATTN_ERR_UNSUPPORTED;
    return FVATTN_OK;
}

namespace fv {

// Curve index of tile (tf_, ty_, tx_) on the 3-D Hilbert curve of a 2^bits
// cube (J. Skilling, "Programming the Hilbert curve", AIP Conf. Proc. 707,
// 2004): undo the curve's rotations and reflections from the top bit down,
// Gray-encode the result, then interleave its bits (frame axis first).
__device__ unsigned long long hilbert_index3(unsigned tf_, unsigned ty_, unsigned tx_, int bits) {
    unsigned a[3] = {tf_, ty_, tx_};
    for (int level = bits - 1; level >= 1; --level) {
        const unsigned q = 1u << level, mask = q - 1u;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            if (a[i] & q) {
                a[0] ^= mask;
            } else {
                const unsigned swap = (a[0] ^ a[i]) & mask;
                a[0] ^= swap;
                a[i] ^= swap;
            }
        }
    }
    a[1] ^= a[0];
    a[2] ^= a[1];
    unsigned flip = 0u;
    for (int level = bits - 1; level >= 1; --level)
        if (a[2] & (1u << level)) flip ^= (1u << level) - 1u;
    unsigned long long key = 0ull;
    for (int level = bits - 1; level >= 0; --level) {
        key = (key << 3) | (static_cast<unsigned long long>(((a[0] ^ flip) >> level) & 1u) << 2) |
              (static_cast<unsigned long long>(((a[1] ^ flip) >> level) & 1u) << 1) |
              static_cast<unsigned long long>(((a[2] ^ flip) >> level) & 1u);
    }
    return key;
}

// One CTA: every tile's curve index into shared memory, then each tile's
// block = its rank among them (indices are distinct).
__global__ void __launch_bounds__(512) block_order_kernel(int nbf, int nby, int nbx, int bits,
                                                          int32_t* __restrict__ table) {
    extern __shared__ unsigned long long curve_key[];
    const int nb = nbf * nby * nbx;
    for (int t = threadIdx.x; t < nb; t += blockDim.x)
        curve_key[t] = hilbert_index3(static_cast<unsigned>(t / (nby * nbx)), static_cast<unsigned>((t / nbx) % nby),
                                      static_cast<unsigned>(t % nbx), bits);
    __syncthreads();
    for (int t = threadIdx.x; t < nb; t += blockDim.x) {
        const unsigned long long k = curve_key[t];
        int rank = 0;
        for (int u = 0; u < nb; ++u) rank += curve_key[u] < k;
        table[rank] = t;
        table[nb + t] = rank;
    }
}

}  // namespace fv

extern "C" int fvattn_block_order(const fvattn_geom* g, int32_t* table, fvattn_stream_t stream) {
    if (!g || !table || (reinterpret_cast<uintptr_t>(table) & 15u) != 0) return FVATTN_ERR_INVALID;
    if (g->nb <= 0 || g->nb > 2560 || g->nbf * g->nby * g->nbx != g->nb) return FVATTN_ERR_INVALID;
    int side = g->nbf > g->nby ? g->nbf : g->nby;
    if (g->nbx > side) side = g->nbx;
    int bits = 1;
    while ((1 << bits) < side) ++bits;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    block_order_kernel<<<1, 512, sizeof(unsigned long long) * g->nb, s>>>(g->nbf, g->nby, g->nbx, bits, table);
    FV_CHECK_LAUNCH();
    return FVATTN_OK;
}

extern "C" int fvattn_get_status(fvattn_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return FVATTN_ERR_CUDA;
    // both words are read and cleared; the attention kernels' error is reported first
    const int va = take_status_attn();
    const int vr = take_status_route();
    return va != FVATTN_OK ? va : vr;
}

extern "C" const char* fvattn_status_string(int code) {
    switch (code) {
        case FVATTN_OK: return "ok";
        case FVATTN_ERR_INVALID: return "invalid argument";
        case FVATTN_ERR_UNSUPPORTED: return "unsupported geometry";
        case FVATTN_ERR_CUDA: return "CUDA error";
        case FVATTN_ERR_TIMEOUT: return "device wait timed out";
        case FVATTN_ERR_BOUNDS: return "kv index or count out of range";
        default: return "unknown status";
    }
}

extern "C" int fvattn_copy_heads(const fvattn_geom* g, int h0, int nh, const void* src, void* dst, int to_device,
                                 fvattn_stream_t stream) {
    if (!g || !src || !dst || h0 < 0 || nh < 1 || h0 + nh > g->H) return FVATTN_ERR_INVALID;
    const size_t row = static_cast<size_t>(g->D) * 2;   // one head of one token, bf16
    const size_t full = row * g->H, part = row * nh;
    const size_t rows = static_cast<size_t>(g->B) * static_cast<size_t>(g->N);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (to_device)
        e = cudaMemcpy2DAsync(dst, part, static_cast<const char*>(src) + row * h0, full, part, rows,
                              cudaMemcpyHostToDevice, s);
    else
        e = cudaMemcpy2DAsync(static_cast<char*>(dst) + row * h0, full, src, part, part, rows,
                              cudaMemcpyDeviceToHost, s);
    return e == cudaSuccess ? FVATTN_OK : FVATTN_ERR_CUDA;
}