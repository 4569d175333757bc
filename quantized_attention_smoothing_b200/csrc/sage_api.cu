// sage_api.cu -- the C ABI of libsage (declared in include/sage.h):
// argument validation, workspace sizing, the Hadamard handle and kernel
// launches. Nothing here allocates per call or synchronises a stream
// (sage_device_error excepted).
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/sage.h"
#include "sage_internal.h"

// The rotation is applied by the kernels as the butterfly x -> x H, whose
// add / subtract pattern is H itself, so no kernel reads the matrix: the
// handle keeps it on the host (for sage_hadamard_matrix) together with the
// device it was built for, which every call checks.
struct sage_hadamard_s {
    int D;
    int device;
    int8_t* host;      // D x D, +-1, row-major
};

namespace sage {

void* tensor_map_encoder() {
    static void* fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = p;
    });
    return fn;
}

}  // namespace sage

namespace {

using sage::View4;

View4 to_view(const sage_cview4& v) {
    View4 r;
    r.ptr = v.ptr;
    for (int i = 0; i < 4; ++i) {
        r.size[i] = v.size[i];
        r.stride[i] = v.stride[i];
    }
    return r;
}

bool sizes_ok(const int64_t* size, const int64_t* stride) {
    for (int i = 0; i < 4; ++i) {
        if (size[i] < 1 || size[i] > (int64_t(1) << 31) - 1) return false;
        if (stride[i] < 0) return false;
    }
    return true;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool blk_ok(int blk) { return blk == 32 || blk == 64 || blk == 128; }

bool current_device(int* dev) { return cudaGetDevice(dev) == cudaSuccess; }

sage_status launch_status(cudaError_t e) { return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA; }

// Checks shared by the decode entry points and the DecodeArgs they fill
// (everything but the cache formats).
sage_status decode_args(sage_hadamard h, sage_cview4 q_bf16, const int32_t* page_table,
                        const int32_t* ctx_lens, int B, int T, int H, int Hk, int D, int page_size,
                        int max_pages, int num_pages, int window, float softmax_scale,
                        sage_view4 out_bf16, uint8_t* q8_out, float* q_scale_out, void* ws,
                        size_t ws_bytes, sage::DecodeArgs* a) {
    if (!h || !q_bf16.ptr || !page_table || !ctx_lens || !out_bf16.ptr) return SAGE_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1 || Hk < 1 || D < 1 || page_size < 1 || max_pages < 1 ||
        num_pages < 1 || window < 1 || !std::isfinite(softmax_scale))
        return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(q_bf16.size, q_bf16.stride) || !sizes_ok(out_bf16.size, out_bf16.stride))
        return SAGE_ERR_INVALID_ARG;
    const int64_t want[4] = {B, T, H, D};
    for (int i = 0; i < 4; ++i)
        if (q_bf16.size[i] != want[i] || out_bf16.size[i] != want[i]) return SAGE_ERR_INVALID_ARG;
    if (D != h->D) return SAGE_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
    if (H % Hk != 0 || H / Hk > 16 || T * (H / Hk) > 64) return SAGE_ERR_UNSUPPORTED;
    if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128)
        return SAGE_ERR_UNSUPPORTED;
    if ((int64_t)num_pages * Hk * page_size * D >= (int64_t(1) << 40)) return SAGE_ERR_UNSUPPORTED;
    if (!aligned(page_table, 4) || !aligned(ctx_lens, 4) || !aligned(q_bf16.ptr, 2) ||
        !aligned(out_bf16.ptr, 2) || !aligned(q8_out, 16) || !aligned(q_scale_out, 4))
        return SAGE_ERR_ALIGNMENT;
    const size_t need = sage::decode_ws_bytes(B, T, H, Hk, D, window);
    if (need > 0 && (!ws || ws_bytes < need)) return SAGE_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return SAGE_ERR_ALIGNMENT;
    int dev = -1;
    if (!current_device(&dev)) return SAGE_ERR_CUDA;
    if (dev != h->device) return SAGE_ERR_INVALID_ARG;
    a->q = to_view(q_bf16);
    a->page_table = page_table;
    a->ctx_lens = ctx_lens;
    a->B = B;
    a->T = T;
    a->H = H;
    a->Hk = Hk;
    a->D = D;
    a->page_size = page_size;
    a->max_pages = max_pages;
    a->num_pages = num_pages;
    a->window = window;
    a->softmax_scale = softmax_scale;
    a->out = out_bf16.ptr;
    for (int i = 0; i < 4; ++i) a->out_stride[i] = out_bf16.stride[i];
    a->ws = ws;
    a->q8_out = q8_out;
    a->q_scale_out = q_scale_out;
    return SAGE_OK;
}


}  // namespace

extern "C" {

const char* sage_status_string(sage_status s) {
    switch (s) {
        case SAGE_OK: return "SAGE_OK";
        case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
        case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
        case SAGE_ERR_ALIGNMENT: return "SAGE_ERR_ALIGNMENT";
        case SAGE_ERR_WORKSPACE: return "SAGE_ERR_WORKSPACE";
        case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
        case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
    }
    return "SAGE_ERR_UNKNOWN";
}

sage_status sage_hadamard_init(int head_dim, int device, sage_hadamard* out) {
    if (out == nullptr || device < 0) return SAGE_ERR_INVALID_ARG;
    *out = nullptr;
    if (head_dim != 64 && head_dim != 128) return SAGE_ERR_UNSUPPORTED;
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess) return SAGE_ERR_CUDA;
    if (device >= count) return SAGE_ERR_INVALID_ARG;
    const int D = head_dim;
    sage_hadamard_s* h = new (std::nothrow) sage_hadamard_s;
    if (!h) return SAGE_ERR_CUDA;
    h->D = D;
    h->device = device;
    h->host = static_cast<int8_t*>(std::malloc((size_t)D * D));
    if (!h->host) {
        delete h;
        return SAGE_ERR_CUDA;
    }
    // Sylvester: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]
    h->host[0] = 1;
    for (int n = 1; n < D; n *= 2)
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                const int8_t v = h->host[i * D + j];
                h->host[i * D + j + n] = v;
                h->host[(i + n) * D + j] = v;
                h->host[(i + n) * D + j + n] = static_cast<int8_t>(-v);
            }
    // H H^T = D I must hold exactly
    for (int i = 0; i < D; ++i)
        for (int j = 0; j < D; ++j) {
            int acc = 0;
            for (int k = 0; k < D; ++k) acc += h->host[i * D + k] * h->host[j * D + k];
            if (acc != (i == j ? D : 0)) {
                std::free(h->host);
                delete h;
                return SAGE_ERR_CUDA;
            }
        }
    *out = h;
    return SAGE_OK;
}

sage_status sage_hadamard_destroy(sage_hadamard h) {
    if (!h) return SAGE_OK;
    std::free(h->host);
    delete h;
    return SAGE_OK;
}

sage_status sage_hadamard_matrix(sage_hadamard h, int8_t* host_out, int* head_dim) {
    if (!h) return SAGE_ERR_INVALID_ARG;
    if (head_dim) *head_dim = h->D;
    if (host_out) std::memcpy(host_out, h->host, (size_t)h->D * h->D);
    return SAGE_OK;
}

size_t sage_quant_qk_workspace(int B, int H, int Hk, int Lq, int Lk, int D) {
    (void)H;
    (void)Lq;
    if (B < 1 || Hk < 1 || Lk < 1 || D < 1) return 0;
    return sage::quant_qk_ws_bytes(B, Hk, Lk, D);
}

sage_status sage_quant_qk(sage_hadamard h, sage_cview4 q_bf16, sage_cview4 k_bf16, int blk_q,
                          int blk_k, int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                          float* k_mean, void* ws, size_t ws_bytes, void* stream) {
    if (!h || !q_bf16.ptr || !k_bf16.ptr || !q8 || !q_scale || !k8 || !k_scale)
        return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(q_bf16.size, q_bf16.stride) || !sizes_ok(k_bf16.size, k_bf16.stride))
        return SAGE_ERR_INVALID_ARG;
    const int64_t B = q_bf16.size[0], H = q_bf16.size[1], Lq = q_bf16.size[2], D = q_bf16.size[3];
    const int64_t Hk = k_bf16.size[1], Lk = k_bf16.size[2];
    if (k_bf16.size[0] != B || k_bf16.size[3] != D) return SAGE_ERR_INVALID_ARG;
    if (D != h->D) return SAGE_ERR_INVALID_ARG;
    if (H % Hk != 0) return SAGE_ERR_UNSUPPORTED;
    if (!blk_ok(blk_q) || !blk_ok(blk_k)) return SAGE_ERR_UNSUPPORTED;
    if (B * H * sage::round_up(Lq, 128) >= (int64_t(1) << 31) ||
        B * Hk * sage::round_up(Lk, 128) >= (int64_t(1) << 31))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(q_scale, 4) || !aligned(k_scale, 4) ||
        !aligned(k_mean, 4) || !aligned(q_bf16.ptr, 2) || !aligned(k_bf16.ptr, 2))
        return SAGE_ERR_ALIGNMENT;
    const size_t need = sage::quant_qk_ws_bytes((int)B, (int)Hk, (int)Lk, (int)D);
    if (need > 0 && (!ws || ws_bytes < need)) return SAGE_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return SAGE_ERR_ALIGNMENT;
    int dev = -1;
    if (!current_device(&dev)) return SAGE_ERR_CUDA;
    if (dev != h->device) return SAGE_ERR_INVALID_ARG;
    return launch_status(sage::launch_quant_qk(to_view(q_bf16), to_view(k_bf16), blk_q, blk_k, q8,
                                               q_scale, k8, k_scale, k_mean, ws,
                                               static_cast<cudaStream_t>(stream)));
}

sage_status sage_quant_k(sage_hadamard h, sage_cview4 k_bf16, int blk_k, int8_t* k8,
                         float* k_scale, float* k_mean, void* ws, size_t ws_bytes, void* stream) {
    if (!h || !k_bf16.ptr || !k8 || !k_scale) return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(k_bf16.size, k_bf16.stride)) return SAGE_ERR_INVALID_ARG;
    const int64_t B = k_bf16.size[0], Hk = k_bf16.size[1], Lk = k_bf16.size[2], D = k_bf16.size[3];
    if (D != h->D) return SAGE_ERR_INVALID_ARG;
    if (!blk_ok(blk_k)) return SAGE_ERR_UNSUPPORTED;
    if (B * Hk * sage::round_up(Lk, 128) >= (int64_t(1) << 31)) return SAGE_ERR_UNSUPPORTED;
    if (!aligned(k8, 16) || !aligned(k_scale, 4) || !aligned(k_mean, 4) || !aligned(k_bf16.ptr, 2))
        return SAGE_ERR_ALIGNMENT;
    const size_t need = sage::quant_qk_ws_bytes((int)B, (int)Hk, (int)Lk, (int)D);
    if (need > 0 && (!ws || ws_bytes < need)) return SAGE_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return SAGE_ERR_ALIGNMENT;
    int dev = -1;
    if (!current_device(&dev)) return SAGE_ERR_CUDA;
    if (dev != h->device) return SAGE_ERR_INVALID_ARG;
    const sage::View4 kv = to_view(k_bf16);
    return launch_status(sage::launch_quant_qk(kv, kv, blk_k, blk_k, nullptr, nullptr, k8, k_scale,
                                               k_mean, ws, static_cast<cudaStream_t>(stream), false));
}

size_t sage_quant_v_workspace(int B, int Hk, int L, int D) {
    if (B < 1 || Hk < 1 || L < 1 || D < 1) return 0;
    return sage::quant_v_ws_bytes(B, Hk, L, D);
}

sage_status sage_quant_v(sage_cview4 v_bf16, uint8_t* v8_t, float* v_scale, void* ws,
                         size_t ws_bytes, void* stream) {
    if (!v_bf16.ptr || !v8_t || !v_scale) return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(v_bf16.size, v_bf16.stride)) return SAGE_ERR_INVALID_ARG;
    const int64_t B = v_bf16.size[0], Hk = v_bf16.size[1], L = v_bf16.size[2], D = v_bf16.size[3];
    if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
    if (B * Hk * D >= (int64_t(1) << 31) || sage::round_up(L, 128) >= (int64_t(1) << 31))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned(v8_t, 16) || !aligned(v_scale, 4) || !aligned(v_bf16.ptr, 2))
        return SAGE_ERR_ALIGNMENT;
    const size_t need = sage::quant_v_ws_bytes((int)B, (int)Hk, (int)L, (int)D);
    if (need > 0 && (!ws || ws_bytes < need)) return SAGE_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return SAGE_ERR_ALIGNMENT;
    return launch_status(sage::launch_quant_v(to_view(v_bf16), v8_t, v_scale, ws,
                                              static_cast<cudaStream_t>(stream)));
}

size_t sage_quant_qkv_workspace(int B, int H, int Hk, int Lq, int Lk, int D) {
    (void)H;
    (void)Lq;
    if (B < 1 || Hk < 1 || Lk < 1 || D < 1) return 0;
    return sage::quant_qkv_ws_bytes(B, Hk, Lk, D);
}

sage_status sage_quant_qkv(sage_hadamard h, sage_cview4 q_bf16, sage_cview4 k_bf16,
                           sage_cview4 v_bf16, int blk_q, int blk_k, int8_t* q8, float* q_scale,
                           int8_t* k8, float* k_scale, float* k_mean, uint8_t* v8_t,
                           float* v_scale, void* ws, size_t ws_bytes, void* stream) {
    if (!h || !q_bf16.ptr || !k_bf16.ptr || !v_bf16.ptr || !q8 || !q_scale || !k8 || !k_scale ||
        !v8_t || !v_scale)
        return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(q_bf16.size, q_bf16.stride) || !sizes_ok(k_bf16.size, k_bf16.stride) ||
        !sizes_ok(v_bf16.size, v_bf16.stride))
        return SAGE_ERR_INVALID_ARG;
    const int64_t B = q_bf16.size[0], H = q_bf16.size[1], Lq = q_bf16.size[2], D = q_bf16.size[3];
    const int64_t Hk = k_bf16.size[1], Lk = k_bf16.size[2];
    if (k_bf16.size[0] != B || k_bf16.size[3] != D) return SAGE_ERR_INVALID_ARG;
    for (int i = 0; i < 4; ++i)
        if (v_bf16.size[i] != k_bf16.size[i]) return SAGE_ERR_INVALID_ARG;
    if (D != h->D) return SAGE_ERR_INVALID_ARG;
    if (H % Hk != 0) return SAGE_ERR_UNSUPPORTED;
    if (!blk_ok(blk_q) || !blk_ok(blk_k)) return SAGE_ERR_UNSUPPORTED;
    if (B * H * sage::round_up(Lq, 128) >= (int64_t(1) << 31) ||
        B * Hk * sage::round_up(Lk, 128) >= (int64_t(1) << 31))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8_t, 16) || !aligned(q_scale, 4) ||
        !aligned(k_scale, 4) || !aligned(k_mean, 4) || !aligned(v_scale, 4) ||
        !aligned(q_bf16.ptr, 2) || !aligned(k_bf16.ptr, 2) || !aligned(v_bf16.ptr, 2))
        return SAGE_ERR_ALIGNMENT;
    const size_t need = sage::quant_qkv_ws_bytes((int)B, (int)Hk, (int)Lk, (int)D);
    if (need > 0 && (!ws || ws_bytes < need)) return SAGE_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return SAGE_ERR_ALIGNMENT;
    int dev = -1;
    if (!current_device(&dev)) return SAGE_ERR_CUDA;
    if (dev != h->device) return SAGE_ERR_INVALID_ARG;
    return launch_status(sage::launch_quant_qkv(to_view(q_bf16), to_view(k_bf16), to_view(v_bf16),
                                                blk_q, blk_k, q8, q_scale, k8, k_scale, k_mean, v8_t,
                                                v_scale, ws, static_cast<cudaStream_t>(stream)));
}

size_t sage_attn_fwd_workspace(int B, int H, int Hk, int Lq, int Lk, int D) {
    (void)B;
    (void)H;
    (void)Hk;
    (void)Lq;
    (void)Lk;
    (void)D;
    return 0;
}

sage_status sage_attn_fwd(const int8_t* q8, const float* q_scale, const int8_t* k8,
                          const float* k_scale, const uint8_t* v8_t, const float* v_scale, int B,
                          int H, int Hk, int Lq, int Lk, int D, int blk_q, int blk_k,
                          float softmax_scale, int causal, sage_view4 out_bf16, void* ws,
                          size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    if (!q8 || !q_scale || !k8 || !k_scale || !v8_t || !v_scale || !out_bf16.ptr)
        return SAGE_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || Hk < 1 || Lq < 1 || Lk < 1 || D < 1) return SAGE_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(out_bf16.size, out_bf16.stride)) return SAGE_ERR_INVALID_ARG;
    if (out_bf16.size[0] != B || out_bf16.size[1] != H || out_bf16.size[2] != Lq ||
        out_bf16.size[3] != D)
        return SAGE_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
    if (H % Hk != 0 || !blk_ok(blk_q) || !blk_ok(blk_k)) return SAGE_ERR_UNSUPPORTED;
    const int64_t nqt = sage::ceil_div(Lq, 256);
    if ((int64_t)B * H > 65535 || nqt > 65535) return SAGE_ERR_UNSUPPORTED;
    if ((int64_t)B * H * sage::round_up(Lq, 128) >= (int64_t(1) << 31) ||
        (int64_t)B * Hk * sage::round_up(Lk, 128) >= (int64_t(1) << 31) ||
        (int64_t)B * Hk * D >= (int64_t(1) << 31))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8_t, 16) || !aligned(q_scale, 4) ||
        !aligned(k_scale, 4) || !aligned(v_scale, 4) || !aligned(out_bf16.ptr, 2))
        return SAGE_ERR_ALIGNMENT;
    sage::AttnArgs a;
    a.q8 = q8;
    a.q_scale = q_scale;
    a.k8 = k8;
    a.k_scale = k_scale;
    a.v8t = v8_t;
    a.v_scale = v_scale;
    a.B = B;
    a.H = H;
    a.Hk = Hk;
    a.Lq = Lq;
    a.Lk = Lk;
    a.D = D;
    a.blk_q = blk_q;
    a.blk_k = blk_k;
    a.softmax_scale = softmax_scale;
    a.causal = causal ? 1 : 0;
    a.out = out_bf16.ptr;
    for (int i = 0; i < 4; ++i) {
        a.out_size[i] = out_bf16.size[i];
        a.out_stride[i] = out_bf16.stride[i];
    }
    if (!sage::tensor_map_encoder()) return SAGE_ERR_CUDA;
    return launch_status(sage::launch_attn_fwd(a, static_cast<cudaStream_t>(stream)));
}

sage_status sage_attn_fwd_q16(sage_hadamard h, sage_cview4 q_bf16, int blk_q, const int8_t* k8,
                              const float* k_scale, const uint8_t* v8_t, const float* v_scale,
                              int Hk, int Lk, int blk_k, float softmax_scale, int causal,
                              sage_view4 out_bf16, void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    if (!h || !q_bf16.ptr || !k8 || !k_scale || !v8_t || !v_scale || !out_bf16.ptr)
        return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(q_bf16.size, q_bf16.stride) || !sizes_ok(out_bf16.size, out_bf16.stride))
        return SAGE_ERR_INVALID_ARG;
    const int64_t B = q_bf16.size[0], H = q_bf16.size[1], Lq = q_bf16.size[2], D = q_bf16.size[3];
    if (Hk < 1 || Lk < 1 || !std::isfinite(softmax_scale)) return SAGE_ERR_INVALID_ARG;
    for (int i = 0; i < 4; ++i)
        if (out_bf16.size[i] != q_bf16.size[i]) return SAGE_ERR_INVALID_ARG;
    if (D != h->D) return SAGE_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
    if (H % Hk != 0 || !blk_ok(blk_q) || !blk_ok(blk_k)) return SAGE_ERR_UNSUPPORTED;
    const int64_t nqt = sage::ceil_div(Lq, 256);
    if (B * H > 65535 || nqt > 65535) return SAGE_ERR_UNSUPPORTED;
    if (B * H * sage::round_up(Lq, 128) >= (int64_t(1) << 31) ||
        B * Hk * sage::round_up(Lk, 128) >= (int64_t(1) << 31) || B * Hk * D >= (int64_t(1) << 31))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned(k8, 16) || !aligned(v8_t, 16) || !aligned(k_scale, 4) || !aligned(v_scale, 4) ||
        !aligned(q_bf16.ptr, 2) || !aligned(out_bf16.ptr, 2))
        return SAGE_ERR_ALIGNMENT;
    int dev = -1;
    if (!current_device(&dev)) return SAGE_ERR_CUDA;
    if (dev != h->device) return SAGE_ERR_INVALID_ARG;
    sage::AttnArgs a;
    a.q8 = nullptr;
    a.q_scale = nullptr;
    a.k8 = k8;
    a.k_scale = k_scale;
    a.v8t = v8_t;
    a.v_scale = v_scale;
    a.B = (int)B;
    a.H = (int)H;
    a.Hk = Hk;
    a.Lq = (int)Lq;
    a.Lk = Lk;
    a.D = (int)D;
    a.blk_q = blk_q;
    a.blk_k = blk_k;
    a.softmax_scale = softmax_scale;
    a.causal = causal ? 1 : 0;
    a.out = out_bf16.ptr;
    for (int i = 0; i < 4; ++i) {
        a.out_size[i] = out_bf16.size[i];
        a.out_stride[i] = out_bf16.stride[i];
    }
    a.qfused = 1;
    a.q16 = to_view(q_bf16);
    if (!sage::tensor_map_encoder()) return SAGE_ERR_CUDA;
    return launch_status(sage::launch_attn_fwd(a, static_cast<cudaStream_t>(stream)));
}

sage_status sage_quant_qk_mx(sage_hadamard h, sage_cview4 q_bf16, sage_cview4 k_bf16, uint8_t* q4,
                             uint8_t* q_sf, uint8_t* k4, uint8_t* k_sf, float* k_mean, void* ws,
                             size_t ws_bytes, void* stream) {
    if (!h || !q_bf16.ptr || !k_bf16.ptr || !q4 || !q_sf || !k4 || !k_sf) return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(q_bf16.size, q_bf16.stride) || !sizes_ok(k_bf16.size, k_bf16.stride))
        return SAGE_ERR_INVALID_ARG;
    const int64_t B = q_bf16.size[0], H = q_bf16.size[1], Lq = q_bf16.size[2], D = q_bf16.size[3];
    const int64_t Hk = k_bf16.size[1], Lk = k_bf16.size[2];
    if (k_bf16.size[0] != B || k_bf16.size[3] != D) return SAGE_ERR_INVALID_ARG;
    if (D != h->D) return SAGE_ERR_INVALID_ARG;
    if (H % Hk != 0) return SAGE_ERR_UNSUPPORTED;
    if (B * H * sage::round_up(Lq, 128) >= (int64_t(1) << 31) ||
        B * Hk * sage::round_up(Lk, 128) >= (int64_t(1) << 31))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned(q4, 16) || !aligned(k4, 16) || !aligned(q_sf, 16) || !aligned(k_sf, 16) ||
        !aligned(k_mean, 4) || !aligned(q_bf16.ptr, 2) || !aligned(k_bf16.ptr, 2))
        return SAGE_ERR_ALIGNMENT;
    const size_t need = sage::quant_qk_ws_bytes((int)B, (int)Hk, (int)Lk, (int)D);
    if (need > 0 && (!ws || ws_bytes < need)) return SAGE_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return SAGE_ERR_ALIGNMENT;
    int dev = -1;
    if (!current_device(&dev)) return SAGE_ERR_CUDA;
    if (dev != h->device) return SAGE_ERR_INVALID_ARG;
    return launch_status(sage::launch_quant_qk_mx(to_view(q_bf16), to_view(k_bf16), q4, q_sf, k4, k_sf,
                                                  k_mean, ws, static_cast<cudaStream_t>(stream)));
}

sage_status sage_attn_fwd_mx(const uint8_t* q4, const uint8_t* q_sf, const uint8_t* k4,
                             const uint8_t* k_sf, const uint8_t* v8_t, const float* v_scale, int B,
                             int H, int Hk, int Lq, int Lk, int D, float softmax_scale, int causal,
                             sage_view4 out_bf16, void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    if (!q4 || !q_sf || !k4 || !k_sf || !v8_t || !v_scale || !out_bf16.ptr) return SAGE_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || Hk < 1 || Lq < 1 || Lk < 1 || D < 1) return SAGE_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.0f)) return SAGE_ERR_INVALID_ARG;
    if (!sizes_ok(out_bf16.size, out_bf16.stride)) return SAGE_ERR_INVALID_ARG;
    if (out_bf16.size[0] != B || out_bf16.size[1] != H || out_bf16.size[2] != Lq || out_bf16.size[3] != D)
        return SAGE_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
    if (H % Hk != 0) return SAGE_ERR_UNSUPPORTED;
    const int64_t nqt = sage::ceil_div(Lq, 128);
    if ((int64_t)B * H > 65535 || nqt > 65535) return SAGE_ERR_UNSUPPORTED;
    if ((int64_t)B * H * sage::round_up(Lq, 128) >= (int64_t(1) << 31) ||
        (int64_t)B * Hk * sage::round_up(Lk, 128) >= (int64_t(1) << 31) ||
        (int64_t)B * Hk * D >= (int64_t(1) << 31))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned(q4, 16) || !aligned(k4, 16) || !aligned(q_sf, 16) || !aligned(k_sf, 16) ||
        !aligned(v8_t, 16) || !aligned(v_scale, 4) || !aligned(out_bf16.ptr, 2))
        return SAGE_ERR_ALIGNMENT;
    sage::AttnMxArgs a;
    a.q4 = q4;
    a.q_sf = q_sf;
    a.k4 = k4;
    a.k_sf = k_sf;
    a.v8t = v8_t;
    a.v_scale = v_scale;
    a.B = B;
    a.H = H;
    a.Hk = Hk;
    a.Lq = Lq;
    a.Lk = Lk;
    a.D = D;
    a.softmax_scale = softmax_scale;
    a.causal = causal ? 1 : 0;
    a.out = out_bf16.ptr;
    for (int i = 0; i < 4; ++i) a.out_stride[i] = out_bf16.stride[i];
    if (!sage::tensor_map_encoder()) return SAGE_ERR_CUDA;
    return launch_status(sage::launch_attn_mx(a, static_cast<cudaStream_t>(stream)));
}

size_t sage_attn_decode_workspace(int B, int T, int H, int Hk, int D, int window) {
    if (B < 1 || T < 1 || H < 1 || Hk < 1 || D < 1 || window < 1) return 0;
    return sage::decode_ws_bytes(B, T, H, Hk, D, window);
}

sage_status sage_attn_decode(sage_hadamard h, sage_cview4 q_bf16, const uint8_t* k_cache,
                             const uint8_t* v_cache, const float* k_scale, const float* v_scale,
                             const int32_t* page_table, const int32_t* ctx_lens, int B, int T,
                             int H, int Hk, int D, int page_size, int max_pages, int num_pages,
                             int window, float softmax_scale, int kv_flags, sage_view4 out_bf16,
                             uint8_t* q8_out, float* q_scale_out, void* ws, size_t ws_bytes,
                             void* stream) {
    if (!k_cache || !v_cache || !k_scale || !v_scale) return SAGE_ERR_INVALID_ARG;
    if (kv_flags & ~(SAGE_KV_PER_TENSOR_SCALES | SAGE_KV_V_TRANSPOSED)) return SAGE_ERR_INVALID_ARG;
    sage::DecodeArgs a;
    sage_status st = decode_args(h, q_bf16, page_table, ctx_lens, B, T, H, Hk, D, page_size, max_pages,
                                 num_pages, window, softmax_scale, out_bf16, q8_out, q_scale_out, ws,
                                 ws_bytes, &a);
    if (st != SAGE_OK) return st;
    if ((kv_flags & SAGE_KV_V_TRANSPOSED) && page_size != 128) return SAGE_ERR_UNSUPPORTED;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(k_scale, 4) || !aligned(v_scale, 4))
        return SAGE_ERR_ALIGNMENT;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.kv_flags = kv_flags;
    return launch_status(sage::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

sage_status sage_attn_decode_mxfp4(sage_hadamard h, sage_cview4 q_bf16, const uint8_t* k_cache,
                                   const uint8_t* v_cache, const uint8_t* k_sf, const uint8_t* v_sf,
                                   const int32_t* page_table, const int32_t* ctx_lens, int B, int T,
                                   int H, int Hk, int D, int page_size, int max_pages, int num_pages,
                                   int window, float softmax_scale, sage_view4 out_bf16,
                                   uint8_t* q8_out, float* q_scale_out, void* ws, size_t ws_bytes,
                                   void* stream) {
    if (!k_cache || !v_cache || !k_sf || !v_sf) return SAGE_ERR_INVALID_ARG;
    sage::DecodeArgs a;
    sage_status st = decode_args(h, q_bf16, page_table, ctx_lens, B, T, H, Hk, D, page_size, max_pages,
                                 num_pages, window, softmax_scale, out_bf16, q8_out, q_scale_out, ws,
                                 ws_bytes, &a);
    if (st != SAGE_OK) return st;
    if (D != 128) return SAGE_ERR_UNSUPPORTED;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(k_sf, 16) || !aligned(v_sf, 16))
        return SAGE_ERR_ALIGNMENT;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.k_scale = nullptr;
    a.v_scale = nullptr;
    a.kv_flags = 0;
    a.mx = 1;
    a.k_sf = k_sf;
    a.v_sf = v_sf;
    return launch_status(sage::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

sage_status sage_device_error_where(void* stream, int* kernel, int* site) {
    if (kernel) *kernel = 0;
    if (site) *site = 0;
    const cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    // error words of the kernels, in the order of SAGE_KERNEL_* ids 1, 2, 3, 4
    const unsigned words[4] = {sage::read_clear_attn_error(), sage::read_clear_decode_error(),
                               sage::read_clear_probe_error(), sage::read_clear_attn_mx_error()};
    if (e != cudaSuccess) return SAGE_ERR_CUDA;
    sage_status st = SAGE_OK;
    for (int i = 0; i < 4; ++i) {
        const unsigned code = words[i] & 0xFFu;
        sage_status si = SAGE_OK;
        if (code == sage::kErrTimeoutCode) si = SAGE_ERR_TIMEOUT;
        else if (code == sage::kErrRangeCode) si = SAGE_ERR_INVALID_ARG;
        // a timeout outranks a range error; the first kernel in id order wins a tie
        const bool take = si != SAGE_OK && (st == SAGE_OK || (si == SAGE_ERR_TIMEOUT && st != SAGE_ERR_TIMEOUT));
        if (take) {
            st = si;
            if (kernel) *kernel = i + 1;
            if (site) *site = static_cast<int>(words[i] >> 8);
        }
    }
    return st;
}

sage_status sage_device_error(void* stream) { return sage_device_error_where(stream, nullptr, nullptr); }

sage_status sage_wait_probe(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000ull || limit_ns > 10000000000ull) return SAGE_ERR_INVALID_ARG;
    return launch_status(sage::launch_wait_probe(static_cast<unsigned long long>(limit_ns),
                                                 static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
