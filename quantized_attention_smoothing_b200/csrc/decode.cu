// decode.cu -- paged FP8-KV decode (placeholder until the kernel lands):
// the entry point validates and reports SAGE_ERR_UNSUPPORTED.
#include "sage_internal.h"

namespace sage {
namespace {
__device__ unsigned g_decode_err;
constexpr int kSplitKeys = 256;
}  // namespace

size_t decode_ws_bytes(int B, int T, int H, int Hk, int D, int window) {
    const int R = T * (H / Hk);
    const int nsplit = static_cast<int>(ceil_div(window + T - 1, kSplitKeys));
    return (size_t)B * Hk * nsplit * R * (D + 2) * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    (void)a;
    (void)s;
    return cudaErrorNotSupported;
}

unsigned read_clear_decode_error() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_decode_err, sizeof v) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_decode_err, &zero, sizeof zero);
    return v;
}

}  // namespace sage
