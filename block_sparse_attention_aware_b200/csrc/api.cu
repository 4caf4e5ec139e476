// Geometry set-up and the device status word of the FVAttn C ABI.
#include "common.cuh"

namespace fv {
__device__ int g_fvattn_status = 0;
}

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
    if (static_cast<long long>(g->B) * g->H * g->Npad >= (1ll << 31)) return FVATTN_ERR_UNSUPPORTED;
    return FVATTN_OK;
}

extern "C" int fvattn_get_status(fvattn_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return FVATTN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_fvattn_status, sizeof(int)) != cudaSuccess) return FVATTN_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fvattn_status, &zero, sizeof(int)) != cudaSuccess) return FVATTN_ERR_CUDA;
    return v;
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
