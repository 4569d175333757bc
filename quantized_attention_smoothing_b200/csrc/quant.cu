// quant.cu -- K smoothing statistics, fused smooth + Hadamard + INT8
// quantisation of Q and K, and FP8 e4m3 per-channel quantisation of V.
//
// Numerics are a fixed operation graph so that results are bit-identical
// to a plain sequential evaluation (this TU is compiled with -fmad=false,
// and every rounding step uses an explicit _rn intrinsic):
//   mean_K = fp32(fp64 sum / L)           (fp64 partial sums per 512-token
//                                          chunk, then chunks in order)
//   x_s    = x - mean_K                   (fp32, K only)
//   x_hat  = butterfly(x_s)               (fp32, stages h = 1, 2, ..., D/2)
//   a      = max |x_hat| over the block;  s = a / 127;  r = 127 / a
//   code   = clamp(rne(x_hat * r), +-127)
//   V:  a = max |v| per channel; s = a / 448; code = e4m3_rn_sat(v * (448/a))
// Sources: "Sage v2 improvements" (Hadamard built once, any-stride inputs);
// "perf(dsv4): qproj wq_b transpose + serving contract; sparse_attn/indexer
// tuning", sequence diagram (Hadamard -> per-head amax -> scale -> INT8);
// "Sage2 SM89 Temporal Pair Experiment", Candidate (per-channel V scale);
// "[FlyDSL] [Misc] pa_decode: ...", Changes (FP8_MAX of e4m3 = 448).
#include <type_traits>

#include <cuda_bf16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// Load 8 consecutive (along D) bf16 values of one token row as raw bits.
// VEC: one 16-byte load (caller guarantees alignment); else 8 scalar loads.
__device__ __forceinline__ uint4 load_row8(const uint16_t* base, int64_t off, int64_t sd,
                                           bool vec) {
    if (vec) return __ldg(reinterpret_cast<const uint4*>(base + off));
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t lo = __ldg(base + off + (2 * i) * sd);
        uint32_t hi = __ldg(base + off + (2 * i + 1) * sd);
        w[i] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        x[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
}

// ---------------------------------------------------------------- stats
// grid (chunks, B*Hh), 256 threads. MODE 0: fp64 column sums (K mean);
// MODE 1: fp32 column absmax (V scale). One output row of D values per
// (b, h, chunk).
template <int D, int MODE>
__global__ void __launch_bounds__(256) column_stats_kernel(View4 x, int L, void* partial,
                                                           int vec) {
    constexpr int TPR = D / 8;           // threads per token row
    constexpr int RPI = 256 / TPR;       // token rows per iteration
    using Acc = typename std::conditional<MODE == 0, double, float>::type;
    __shared__ Acc red[RPI][D];

    const int Hh = static_cast<int>(x.size[1]);
    const int bh = blockIdx.y;
    const int b = bh / Hh, h = bh % Hh;
    const int tid = threadIdx.x;
    const int cg = tid % TPR, rg = tid / TPR;
    const int l0 = blockIdx.x * kStatRows;
    const int l1 = min(L, l0 + kStatRows);
    const uint16_t* base = static_cast<const uint16_t*>(x.ptr);
    const int64_t row0 = b * x.stride[0] + h * x.stride[1] + (int64_t)(cg * 8) * x.stride[3];

    Acc acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = Acc(0);
    for (int l = l0 + rg; l < l1; l += 4 * RPI) {
        uint4 u[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int ll = l + k * RPI;
            u[k] = ll < l1 ? load_row8(base, row0 + (int64_t)ll * x.stride[2], x.stride[3], vec != 0)
                           : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float v[8];
            unpack8(u[k], v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (MODE == 0) acc[i] = __dadd_rn(acc[i], (double)v[i]);
                else acc[i] = fmaxf(acc[i], fabsf(v[i]));
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[rg][cg * 8 + i] = acc[i];
    __syncthreads();
    if (tid < D) {
        Acc s = red[0][tid];
        for (int r = 1; r < RPI; ++r) {
            if (MODE == 0) s = __dadd_rn(s, red[r][tid]);
            else s = fmaxf(s, red[r][tid]);
        }
        static_cast<Acc*>(partial)[((int64_t)bh * gridDim.x + blockIdx.x) * D + tid] = s;
    }
}

template <int D>
__device__ __forceinline__ void butterfly(float (&x)[D]) {
    // stage h pairs (j, j + h) for j = (k / h) * 2h + k % h, k = 0 .. D/2 - 1
#pragma unroll
    for (int lg = 0; (1 << lg) < D; ++lg) {
        const int h = 1 << lg;
#pragma unroll
        for (int k = 0; k < D / 2; ++k) {
            const int j = ((k >> lg) << (lg + 1)) + (k & (h - 1));
            const float a = x[j], c = x[j + h];
            x[j] = __fadd_rn(a, c);
            x[j + h] = __fsub_rn(a, c);
        }
    }
}

// ---------------------------------------------------------------- Q/K int8
// One CTA per (tensor, b, h, 128-token tile); D/32 threads per token, each
// holding 32 consecutive channels. The butterfly stages h < 32 run inside a
// thread; h = 32 and h = 64 pair lanes (lane ^ 1, lane ^ 2) and every output
// is still the single fp32 add (lower + upper) or subtract (lower - upper)
// of the same two values as in a sequential evaluation.
template <int D>
__global__ void __launch_bounds__(kTile * (D / 32)) qk_quant_kernel(
    View4 q, View4 k, int blk_q, int blk_k, int n_qtiles, const double* __restrict__ ksum,
    int kchunks, int8_t* __restrict__ q8, float* __restrict__ q_scale, int8_t* __restrict__ k8,
    float* __restrict__ k_scale, float* __restrict__ k_mean, int qvec, int kvec) {
    constexpr int TPR = D / 32;                   // threads per token row
    constexpr int NT = kTile * TPR;
    constexpr int NW = NT / 32;                   // warps
    constexpr int RPW = 32 / TPR;                 // rows per warp
    __shared__ float mean_s[D];
    __shared__ float wmax[NW];

    const bool isK = blockIdx.x >= (unsigned)n_qtiles;
    const View4& x = isK ? k : q;
    const int tile_lin = isK ? blockIdx.x - n_qtiles : blockIdx.x;
    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    const int ntiles = static_cast<int>(ceil_div(L, kTile));
    const int bh = tile_lin / ntiles, tl = tile_lin % ntiles;
    const int b = bh / Hh, h = bh % Hh;
    const int blk = isK ? blk_k : blk_q;
    const int nb = static_cast<int>(ceil_div(L, blk));
    const bool vec = (isK ? kvec : qvec) != 0;
    const int tid = threadIdx.x;
    const int r = tid / TPR, c = tid % TPR;
    const int l = tl * kTile + r;
    const bool valid = l < L;

    // issue the row loads first (32 channels = 64 bytes per thread)
    const uint16_t* base = static_cast<const uint16_t*>(x.ptr);
    const int64_t off = b * x.stride[0] + h * x.stride[1] + (int64_t)l * x.stride[2] +
                        (int64_t)(32 * c) * x.stride[3];
    uint4 raw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        raw[i] = valid ? load_row8(base, off + (int64_t)(8 * i) * x.stride[3], x.stride[3], vec)
                       : make_uint4(0, 0, 0, 0);

    if (isK && tid < D) {
        const double* p = ksum + (int64_t)bh * kchunks * D + tid;
        double s = p[0];
        for (int ch = 1; ch < kchunks; ++ch) s = __dadd_rn(s, p[(int64_t)ch * D]);
        const float m = __double2float_rn(__ddiv_rn(s, (double)L));
        mean_s[tid] = m;
        if (tl == 0 && k_mean != nullptr) k_mean[(int64_t)bh * D + tid] = m;
    }
    __syncthreads();

    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float t8[8];
        unpack8(raw[i], t8);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[8 * i + j] = t8[j];
    }
    if (isK && valid) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __fsub_rn(v[j], mean_s[32 * c + j]);
    }
    butterfly<32>(v);
#pragma unroll
    for (int hb = 1; hb < TPR; hb <<= 1) {       // stages h = 32 * hb across lanes
        const bool upper = (c & hb) != 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, v[j], hb);
            v[j] = upper ? __fsub_rn(o, v[j]) : __fadd_rn(v[j], o);
        }
    }

    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) a = fmaxf(a, fabsf(v[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const int warp = tid >> 5;
    if ((tid & 31) == 0) wmax[warp] = a;
    __syncthreads();
    const int wpb = max(1, blk / RPW);            // warps per quantisation block
    const int w0 = (warp / wpb) * wpb;
    float amax = 0.0f;
    for (int w = w0; w < w0 + wpb; ++w) amax = fmaxf(amax, wmax[w]);
    float s = 0.0f, rr = 0.0f;
    if (amax != 0.0f) {
        s = __fdiv_rn(amax, 127.0f);
        rr = __fdiv_rn(127.0f, amax);
    }
    if (valid && c == 0 && (l % blk) == 0) {
        float* scales = isK ? k_scale : q_scale;
        scales[(int64_t)bh * nb + l / blk] = s;
    }
    uint32_t w[8];
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) {
        uint32_t word = 0;
#pragma unroll
        for (int bi = 0; bi < 4; ++bi) {
            int code = __float2int_rn(__fmul_rn(v[4 * wi + bi], rr));
            code = max(-127, min(127, code));
            word |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * bi);
        }
        w[wi] = word;
    }
    int8_t* dst = (isK ? k8 : q8) + ((int64_t)bh * ntiles * kTile + l) * D + 32 * c;
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// ---------------------------------------------------------------- V e4m3
// One CTA of 128 threads per (b, h, 128-token tile). Writes V transposed:
// v8t[b, h, d, token].
template <int D>
__global__ void __launch_bounds__(128) v_quant_kernel(View4 x, const float* __restrict__ vmax,
                                                      int vchunks, uint8_t* __restrict__ v8t,
                                                      float* __restrict__ v_scale, int vec) {
    constexpr int RS = D + 8;
    constexpr int OS = kTile + 16;               // output staging row stride (bytes)
    static_assert(D * OS <= kTile * RS * 2, "output staging reuses the input buffer");
    __shared__ __align__(16) uint16_t stage[kTile * RS];
    __shared__ float rmul[D];

    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    const int ntiles = static_cast<int>(ceil_div(L, kTile));
    const int bh = blockIdx.x / ntiles, tl = blockIdx.x % ntiles;
    const int b = bh / Hh, h = bh % Hh;
    const int tid = threadIdx.x;

    if (tid < D) {
        const float* p = vmax + (int64_t)bh * vchunks * D + tid;
        float a = p[0];
        for (int c = 1; c < vchunks; ++c) a = fmaxf(a, p[(int64_t)c * D]);
        float s = 0.0f, r = 0.0f;
        if (a != 0.0f) {
            s = __fdiv_rn(a, 448.0f);
            r = __fdiv_rn(448.0f, a);
        }
        rmul[tid] = r;
        if (tl == 0) v_scale[(int64_t)bh * D + tid] = s;
    }
    const uint16_t* base = static_cast<const uint16_t*>(x.ptr);
    const int64_t hoff = b * x.stride[0] + h * x.stride[1];
    for (int c = tid; c < kTile * (D / 8); c += 128) {
        const int r = c / (D / 8), cc = c % (D / 8);
        const int l = tl * kTile + r;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (l < L) u = load_row8(base, hoff + (int64_t)l * x.stride[2] + (int64_t)(cc * 8) * x.stride[3],
                                 x.stride[3], vec != 0);
        *reinterpret_cast<uint4*>(&stage[r * RS + cc * 8]) = u;
    }
    __syncthreads();
    uint32_t w[kTile / 4];
    if (tid < D) {
        const float r = rmul[tid];
#pragma unroll
        for (int wi = 0; wi < kTile / 4; ++wi) {
            float y[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                y[i] = __fmul_rn(bf16_bits_to_f32(stage[(wi * 4 + i) * RS + tid]), r);
            const uint32_t lo = e4m3x2_rn_satfinite(y[0], y[1]);
            const uint32_t hi = e4m3x2_rn_satfinite(y[2], y[3]);
            w[wi] = lo | (hi << 16);
        }
    }
    __syncthreads();
    uint8_t* ost = reinterpret_cast<uint8_t*>(stage);
    if (tid < D) {
#pragma unroll
        for (int c = 0; c < kTile / 16; ++c)
            *reinterpret_cast<uint4*>(&ost[tid * OS + c * 16]) =
                make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    }
    __syncthreads();
    const int64_t Lpad = (int64_t)ntiles * kTile;
    uint8_t* dst = v8t + (int64_t)bh * D * Lpad + (int64_t)tl * kTile;
    for (int c = tid; c < D * (kTile / 16); c += 128) {
        const int d = c / (kTile / 16), cc = c % (kTile / 16);
        *reinterpret_cast<uint4*>(dst + (int64_t)d * Lpad + cc * 16) =
            *reinterpret_cast<const uint4*>(&ost[d * OS + cc * 16]);
    }
}

}  // namespace

size_t quant_qk_ws_bytes(int B, int Hk, int Lk, int D) {
    return (size_t)B * Hk * stat_chunks(Lk) * D * sizeof(double);
}

size_t quant_v_ws_bytes(int B, int Hk, int L, int D) {
    return (size_t)B * Hk * stat_chunks(L) * D * sizeof(float);
}

cudaError_t launch_quant_qk(const View4& q, const View4& k, int blk_q, int blk_k, int8_t* q8,
                            float* q_scale, int8_t* k8, float* k_scale, float* k_mean, void* ws,
                            cudaStream_t s) {
    const int B = (int)q.size[0], H = (int)q.size[1], Lq = (int)q.size[2], D = (int)q.size[3];
    const int Hk = (int)k.size[1], Lk = (int)k.size[2];
    const int kchunks = stat_chunks(Lk);
    const int kvec = view_vec8(k), qvec = view_vec8(q);
    double* ksum = static_cast<double*>(ws);
    const dim3 sgrid(kchunks, B * Hk);
    const int n_qtiles = B * H * (int)ceil_div(Lq, kTile);
    const int n_ktiles = B * Hk * (int)ceil_div(Lk, kTile);
    if (D == 128) {
        column_stats_kernel<128, 0><<<sgrid, 256, 0, s>>>(k, Lk, ksum, kvec);
        qk_quant_kernel<128><<<n_qtiles + n_ktiles, kTile * 4, 0, s>>>(
            q, k, blk_q, blk_k, n_qtiles, ksum, kchunks, q8, q_scale, k8, k_scale, k_mean, qvec, kvec);
    } else {
        column_stats_kernel<64, 0><<<sgrid, 256, 0, s>>>(k, Lk, ksum, kvec);
        qk_quant_kernel<64><<<n_qtiles + n_ktiles, kTile * 2, 0, s>>>(
            q, k, blk_q, blk_k, n_qtiles, ksum, kchunks, q8, q_scale, k8, k_scale, k_mean, qvec, kvec);
    }
    return cudaGetLastError();
}

cudaError_t launch_quant_v(const View4& v, uint8_t* v8t, float* v_scale, void* ws,
                           cudaStream_t s) {
    const int B = (int)v.size[0], Hk = (int)v.size[1], L = (int)v.size[2], D = (int)v.size[3];
    const int chunks = stat_chunks(L);
    const int vec = view_vec8(v);
    float* vmax = static_cast<float*>(ws);
    const dim3 sgrid(chunks, B * Hk);
    const int ntiles = B * Hk * (int)ceil_div(L, kTile);
    if (D == 128) {
        column_stats_kernel<128, 1><<<sgrid, 256, 0, s>>>(v, L, vmax, vec);
        v_quant_kernel<128><<<ntiles, 128, 0, s>>>(v, vmax, chunks, v8t, v_scale, vec);
    } else {
        column_stats_kernel<64, 1><<<sgrid, 256, 0, s>>>(v, L, vmax, vec);
        v_quant_kernel<64><<<ntiles, 128, 0, s>>>(v, vmax, chunks, v8t, v_scale, vec);
    }
    return cudaGetLastError();
}

}  // namespace sage

// ---------------------------------------------------------------- no-allocation variant
// sage_quant_qk_noalloc: the same Q/K smoothing + rotation + INT8 quantisation
// as sage_quant_qk, for callers that cannot allocate device memory at the
// point of the call -- for instance a serving loop whose device memory is
// budgeted once at start-up, or code that must not risk the implicit device
// synchronisation that cudaMalloc / cudaFree can cause. Its scratch (the fp64
// per-chunk column sums of K) lives in the fixed array below instead of a
// caller workspace.
#include <mutex>

#include "../../include/sage.h"

namespace {

// Largest scratch the no-allocation entry point supports. Every GPU that
// loads libsage holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;    // 8 MiB
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_qk_noalloc_scratch[kNoAllocScratchBytes];

// Host code cannot use g_qk_noalloc_scratch directly: on the host the name
// stands for a host-side shadow, not a device address. The device address is
// looked up once per device (with that device current) and cached.
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

sage_status noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return SAGE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_qk_noalloc_scratch) != cudaSuccess || p == nullptr)
            return SAGE_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SAGE_OK;
}

}  // namespace

extern "C" sage_status sage_quant_qk_noalloc(sage_hadamard h, sage_cview4 q_bf16,
                                             sage_cview4 k_bf16, int blk_q, int blk_k, int8_t* q8,
                                             float* q_scale, int8_t* k8, float* k_scale,
                                             float* k_mean, void* stream) {
    if (!h || !k_bf16.ptr) return SAGE_ERR_INVALID_ARG;
    const int64_t B = k_bf16.size[0], Hk = k_bf16.size[1], Lk = k_bf16.size[2], D = k_bf16.size[3];
    if (B < 1 || Hk < 1 || Lk < 1 || D < 1 || Lk > (int64_t(1) << 31) - 1) return SAGE_ERR_INVALID_ARG;
    const size_t need = sage::quant_qk_ws_bytes((int)B, (int)Hk, (int)Lk, (int)D);
    if (need > kNoAllocScratchBytes) return SAGE_ERR_WORKSPACE;     // beyond the fixed scratch
    void* scratch = nullptr;
    const sage_status st = noalloc_scratch(&scratch);
    if (st != SAGE_OK) return st;
    return sage_quant_qk(h, q_bf16, k_bf16, blk_q, blk_k, q8, q_scale, k8, k_scale, k_mean, scratch,
                         kNoAllocScratchBytes, stream);
}
