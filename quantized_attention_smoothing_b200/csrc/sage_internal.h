// sage_internal.h -- declarations shared between the C-ABI layer and the
// kernel translation units of libsage. Not installed, not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace sage {

// Plain copy of a caller's view (element sizes / strides), passed by value
// to kernels.
struct View4 {
    const void* ptr;
    int64_t size[4];
    int64_t stride[4];
};

// 16-byte vector access is possible: unit innermost stride, the other
// strides multiples of 8 elements, 16-byte aligned base.
inline bool view_vec8(const View4& v) {
    return v.stride[3] == 1 && (v.stride[0] % 8) == 0 && (v.stride[1] % 8) == 0 &&
           (v.stride[2] % 8) == 0 && (reinterpret_cast<uintptr_t>(v.ptr) % 16) == 0;
}

constexpr int kTile = 128;                  // token tile of every kernel
constexpr unsigned kErrTimeoutCode = 1u;    // low byte of a device error word
constexpr unsigned kErrRangeCode = 2u;      // decode: a page id or context length out of range

__host__ __device__ inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Launch `kern` with programmatic stream serialisation: it may start while
// the preceding kernel of the stream is still running, and must call
// griddepcontrol.wait before touching that kernel's outputs.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Params>(args)...);
}

// Number of SMs of the current device (looked up once per device).
inline int num_sms() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}
__host__ __device__ inline int64_t ceil_div(int64_t x, int64_t m) { return (x + m - 1) / m; }

// ---- quantisation (quant.cu)
size_t quant_qk_ws_bytes(int B, int Hk, int Lk, int D);
size_t quant_v_ws_bytes(int B, int Hk, int L, int D);
// with_q = false: K alone (q, q8, q_scale unused)
cudaError_t launch_quant_qk(const View4& q, const View4& k, int blk_q, int blk_k, int8_t* q8,
                            float* q_scale, int8_t* k8, float* k_scale, float* k_mean,
                            void* ws, cudaStream_t s, bool with_q = true);
cudaError_t launch_quant_v(const View4& v, uint8_t* v8t, float* v_scale, void* ws,
                           cudaStream_t s);
// Q, K and V together (V shaped like K): two launches in all
size_t quant_qkv_ws_bytes(int B, int Hk, int Lk, int D);
cudaError_t launch_quant_qkv(const View4& q, const View4& k, const View4& v, int blk_q, int blk_k,
                             int8_t* q8, float* q_scale, int8_t* k8, float* k_scale, float* k_mean,
                             uint8_t* v8t, float* v_scale, void* ws, cudaStream_t s);

// Q and K as MXFP4 (E2M1 codes, e8m0 scales per 32 elements): two launches
cudaError_t launch_quant_qk_mx(const View4& q, const View4& k, uint8_t* q4, uint8_t* q_sf, uint8_t* k4,
                               uint8_t* k_sf, float* k_mean, void* ws, cudaStream_t s);

// ---- attention forward (attn_fwd.cu)
struct AttnArgs {
    const int8_t* q8;
    const float* q_scale;
    const int8_t* k8;
    const float* k_scale;
    const uint8_t* v8t;
    const float* v_scale;
    int B, H, Hk, Lq, Lk, D, blk_q, blk_k;
    float softmax_scale;
    int causal;
    void* out;
    int64_t out_size[4];
    int64_t out_stride[4];
    // in-CTA Q path: q8 / q_scale unused, Q rotated and quantised from this
    // bf16 [B, H, Lq, D] view inside the attention kernel
    int qfused = 0;
    View4 q16 = {};
};
cudaError_t launch_attn_fwd(const AttnArgs& a, cudaStream_t s);
unsigned read_clear_attn_error();

// ---- MXFP4 attention forward (attn_mx.cu)
struct AttnMxArgs {
    const uint8_t* q4;
    const uint8_t* q_sf;
    const uint8_t* k4;
    const uint8_t* k_sf;
    const uint8_t* v8t;
    const float* v_scale;
    int B, H, Hk, Lq, Lk, D;
    float softmax_scale;
    int causal;
    void* out;
    int64_t out_stride[4];
};
cudaError_t launch_attn_mx(const AttnMxArgs& a, cudaStream_t s);
unsigned read_clear_attn_mx_error();

// ---- decode (decode.cu)
struct DecodeArgs {
    View4 q;                   // [B, T, H, D] bf16
    const uint8_t* k_cache;
    const uint8_t* v_cache;
    const float* k_scale;
    const float* v_scale;
    const int32_t* page_table;
    const int32_t* ctx_lens;
    int B, T, H, Hk, D, page_size, max_pages, num_pages, window;
    float softmax_scale;
    void* out;
    int64_t out_stride[4];
    void* ws;
    uint8_t* q8_out;           // optional [B, T, H, D] e4m3 query codes
    float* q_scale_out;        // optional [B, T, H] query scales
    int kv_flags;              // SAGE_KV_PER_TENSOR_SCALES | SAGE_KV_V_TRANSPOSED
    int mx = 0;                // k_cache / v_cache: E2M1 codes [.., page, D / 2] with
    const uint8_t* k_sf = nullptr;   // e8m0 block scales [num_pages, Hk, page, D / 32]
    const uint8_t* v_sf = nullptr;
};
size_t decode_ws_bytes(int B, int T, int H, int Hk, int D, int window);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
unsigned read_clear_decode_error();

// ---- bounded-wait timeout probe (probe.cu)
cudaError_t launch_wait_probe(unsigned long long limit_ns, cudaStream_t s);
unsigned read_clear_probe_error();

// ---- driver entry point for tensor-map encoding (sage_api.cu)
void* tensor_map_encoder();

}  // namespace sage
