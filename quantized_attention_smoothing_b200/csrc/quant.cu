// quant.cu -- K smoothing statistics, fused smooth + Hadamard + INT8
// quantisation of Q and K, and FP8 e4m3 per-channel quantisation of V.
//
// Numerics are a fixed operation graph so that results are bit-identical
// to a plain sequential evaluation (this TU is compiled with -fmad=false,
// and every rounding step uses an explicit _rn intrinsic):
//   mean_K = fp32(fp64 sum / L)           (fp64 partial sums per CTA, then
//                                          CTAs of the cluster in order)
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
//
// Kernels (each a single pass over its tensor):
//   column_stats_kernel  one cluster of 8 CTAs per (b, h) streams the head's
//                        tokens and reduces the column statistic across the
//                        cluster through distributed shared memory; the
//                        leader CTA writes the finished per-channel values.
//   qk_quant_kernel      one CTA per 128-token tile; the tile's rows arrive in
//                        shared memory by bulk copies, then one thread owns
//                        one token row, so all log2(D) butterfly stages stay
//                        inside a thread.
//   v_quant_kernel       one CTA per 128-token tile, staged the same way,
//                        written out transposed [b, h, d, token].
#include <type_traits>

#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {

__device__ unsigned g_quant_err;

namespace {

namespace cg = cooperative_groups;

constexpr int kStatCluster = 8;      // CTAs per (b, h) in the statistics kernel
constexpr int kStatThreads = 512;
constexpr int kStatUnroll = 8;       // 16-byte loads in flight per thread
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

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

__device__ __forceinline__ void unpack8(const uint4& u, float* x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// ---------------------------------------------------------------- stats
// grid (8 * B*Hh), 512 threads, clusters of 8 along x: CTA `rank` of the
// cluster of head bh covers tokens [rank * span, (rank + 1) * span).
// MODE 0 (K): fp64 column sums -> mean (fp32) into `ws`, and into `user`
//             (the optional k_mean output) when given.
// MODE 1 (V): fp32 column absmax a -> scale a / 448 into `user` (v_scale)
//             and the multiplier 448 / a into `ws`.
template <int D, int MODE>
__global__ void __cluster_dims__(kStatCluster, 1, 1) __launch_bounds__(kStatThreads)
    column_stats_kernel(View4 x, float* __restrict__ ws, float* __restrict__ user, int vec) {
    constexpr int TPR = D / 8;                    // threads per token row
    constexpr int RPI = kStatThreads / TPR;       // token rows per load round
    using Acc = typename std::conditional<MODE == 0, double, float>::type;
    __shared__ Acc red[RPI][D];
    __shared__ Acc part[D];

    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    const int rank = blockIdx.x % kStatCluster;
    const int bh = blockIdx.x / kStatCluster;
    const int b = bh / Hh, h = bh % Hh;
    const int tid = threadIdx.x;
    const int cg8 = tid % TPR, rg = tid / TPR;
    const int span = static_cast<int>(ceil_div(L, kStatCluster));
    const int l0 = rank * span;
    const int l1 = min(L, l0 + span);
    const uint16_t* base = static_cast<const uint16_t*>(x.ptr);
    const int64_t row0 = b * x.stride[0] + h * x.stride[1] + (int64_t)(cg8 * 8) * x.stride[3];

    Acc acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = Acc(0);
    for (int l = l0 + rg; l < l1; l += kStatUnroll * RPI) {
        uint4 u[kStatUnroll];
#pragma unroll
        for (int k = 0; k < kStatUnroll; ++k) {
            const int ll = l + k * RPI;
            u[k] = ll < l1 ? load_row8(base, row0 + (int64_t)ll * x.stride[2], x.stride[3], vec != 0)
                           : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < kStatUnroll; ++k) {
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
    for (int i = 0; i < 8; ++i) red[rg][cg8 * 8 + i] = acc[i];
    __syncthreads();
    if (tid < D) {
        Acc s = red[0][tid];
        for (int r = 1; r < RPI; ++r) {
            if (MODE == 0) s = __dadd_rn(s, red[r][tid]);
            else s = fmaxf(s, red[r][tid]);
        }
        part[tid] = s;
    }
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();
    if (rank == 0 && tid < D) {
        Acc s = part[tid];
        for (int r = 1; r < kStatCluster; ++r) {
            const Acc o = cl.map_shared_rank(part, r)[tid];
            if (MODE == 0) s = __dadd_rn(s, o);
            else s = fmaxf(s, o);
        }
        const int64_t o = (int64_t)bh * D + tid;
        if (MODE == 0) {
            const float m = __double2float_rn(__ddiv_rn(s, (double)L));
            ws[o] = m;
            if (user != nullptr) user[o] = m;
        } else {
            float sc = 0.0f, r = 0.0f;
            if (s != 0.0f) {
                sc = __fdiv_rn(s, 448.0f);
                r = __fdiv_rn(448.0f, s);
            }
            user[o] = sc;
            ws[o] = r;
        }
    }
    cl.sync();                  // the leader has read every CTA's partials
}

// ---------------------------------------------------------------- staging
// The rows [0, nrows) of a 128-token tile of head (b, h), D bf16 each, into
// shared memory at a pitch of D + 8 elements (rows land 16 bytes apart in
// the bank space, so a thread reading its own row conflicts with nobody).
// VEC views: one bulk copy per row, completion on `bar`; other views: a
// strided element gather by the whole CTA. Returns false (and records a
// timeout) if the copies never arrive.
template <int D>
__device__ __forceinline__ bool stage_tile(const View4& x, int b, int h, int l0, int nrows,
                                           bool vec, uint16_t* tile, uint64_t* bar,
                                           volatile int* abort_flag, unsigned site) {
    constexpr int PITCH = D + 8;
    const int tid = threadIdx.x;
    const uint16_t* base = static_cast<const uint16_t*>(x.ptr);
    const int64_t hoff = b * x.stride[0] + h * x.stride[1];
    if (vec) {
        if (tid < 32) {
            if (tid == 0) mbar_arrive_expect_tx(bar, (uint32_t)(nrows * D * 2));
            __syncwarp();
            for (int r = tid; r < nrows; r += 32)
                bulk_load(tile + r * PITCH, base + hoff + (int64_t)(l0 + r) * x.stride[2], D * 2, bar);
        }
        return mbar_wait(bar, 0, abort_flag, &g_quant_err, site);
    }
    for (int i = tid; i < nrows * D; i += kTile) {
        const int r = i / D, d = i % D;
        tile[r * PITCH + d] = __ldg(base + hoff + (int64_t)(l0 + r) * x.stride[2] + (int64_t)d * x.stride[3]);
    }
    __syncthreads();
    return true;
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

// Low byte of the fp32 bit pattern of (y + 1.5 * 2^23) is rne(y) as a two's
// complement byte for |y| < 2^22; four of them into one word.
__device__ __forceinline__ uint32_t pack_round4(float y0, float y1, float y2, float y3) {
    const uint32_t t0 = __float_as_uint(__fadd_rn(y0, kRoundMagic));
    const uint32_t t1 = __float_as_uint(__fadd_rn(y1, kRoundMagic));
    const uint32_t t2 = __float_as_uint(__fadd_rn(y2, kRoundMagic));
    const uint32_t t3 = __float_as_uint(__fadd_rn(y3, kRoundMagic));
    return __byte_perm(__byte_perm(t0, t1, 0x0040), __byte_perm(t2, t3, 0x0040), 0x5410);
}

__device__ __forceinline__ uint32_t pack_clamp4(float y0, float y1, float y2, float y3) {
    const float y[4] = {y0, y1, y2, y3};
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int code = __float2int_rn(y[i]);
        code = max(-127, min(127, code));
        word |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * i);
    }
    return word;
}

// ---------------------------------------------------------------- Q/K int8
// One CTA of 128 threads per (tensor, b, h, 128-token tile); thread r owns
// token row r of the tile. Q tiles come first in the grid, then K tiles.
template <int D>
__global__ void __launch_bounds__(kTile) qk_quant_kernel(
    View4 q, View4 k, int blk_q, int blk_k, int n_qtiles, const float* __restrict__ kmean,
    int8_t* __restrict__ q8, float* __restrict__ q_scale, int8_t* __restrict__ k8,
    float* __restrict__ k_scale, int qvec, int kvec) {
    constexpr int PITCH = D + 8;                  // staged input row pitch (elements)
    constexpr int OPITCH = D + 16;                // staged output row pitch (bytes)
    static_assert(kTile * OPITCH <= kTile * PITCH * 2, "output staging reuses the tile");
    __shared__ __align__(128) uint16_t tile[kTile * PITCH];
    __shared__ __align__(16) float mean_s[D];
    __shared__ float wmax[kTile / 32];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;

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
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l0 = tl * kTile;
    const int nrows = min(kTile, L - l0);

    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (isK && tid < D) mean_s[tid] = kmean[(int64_t)bh * D + tid];
    __syncthreads();
    if (!stage_tile<D>(x, b, h, l0, nrows, vec, tile, &bar, &abort_flag, 1)) return;

    const bool valid = tid < nrows;
    float v[D];
    {
        const uint16_t* row = tile + tid * PITCH;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 u = valid ? *reinterpret_cast<const uint4*>(row + 8 * c) : make_uint4(0, 0, 0, 0);
            unpack8(u, v + 8 * c);
        }
    }
    if (isK && valid) {
#pragma unroll
        for (int c = 0; c < D / 4; ++c) {
            const float4 m = *reinterpret_cast<const float4*>(mean_s + 4 * c);
            v[4 * c] = __fsub_rn(v[4 * c], m.x);
            v[4 * c + 1] = __fsub_rn(v[4 * c + 1], m.y);
            v[4 * c + 2] = __fsub_rn(v[4 * c + 2], m.z);
            v[4 * c + 3] = __fsub_rn(v[4 * c + 3], m.w);
        }
    }
    butterfly<D>(v);

    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < D; ++j) a = fmaxf(a, fabsf(v[j]));
    // a >= +0, so the bit patterns order like the values
    const unsigned am = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
    if (lane == 0) wmax[warp] = __uint_as_float(am);
    __syncthreads();              // every row has left the tile; block maxima are in
    const int wpb = blk / 32;     // warps per quantisation block (blk in {32, 64, 128})
    const int w0 = (warp / wpb) * wpb;
    float amax = 0.0f;
    for (int w = w0; w < w0 + wpb; ++w) amax = fmaxf(amax, wmax[w]);
    float s = 0.0f, rr = 0.0f;
    if (amax != 0.0f) {
        s = __fdiv_rn(amax, 127.0f);
        rr = __fdiv_rn(127.0f, amax);
    }
    const int l = l0 + tid;
    if (valid && (l & (blk - 1)) == 0) {
        float* scales = isK ? k_scale : q_scale;
        scales[(int64_t)bh * nb + l / blk] = s;
    }

    // |x_hat * r| <= a * fl(127 / a) rounds to at most 127 whenever r is
    // finite, so the magic-number rounding needs no clamp; a block whose
    // amax is so small that 127 / a overflows takes the clamped conversion.
    uint8_t* ost = reinterpret_cast<uint8_t*>(tile);
    uint8_t* orow = ost + tid * OPITCH;
    if (isfinite(rr)) {
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
            uint32_t w4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float* p = v + 16 * c + 4 * i;
                w4[i] = pack_round4(__fmul_rn(p[0], rr), __fmul_rn(p[1], rr), __fmul_rn(p[2], rr),
                                    __fmul_rn(p[3], rr));
            }
            *reinterpret_cast<uint4*>(orow + 16 * c) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    } else {
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
            uint32_t w4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float* p = v + 16 * c + 4 * i;
                w4[i] = pack_clamp4(__fmul_rn(p[0], rr), __fmul_rn(p[1], rr), __fmul_rn(p[2], rr),
                                    __fmul_rn(p[3], rr));
            }
            *reinterpret_cast<uint4*>(orow + 16 * c) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
    __syncthreads();
    // the tile's 128 output rows are one contiguous run of 128 * D bytes
    int8_t* dst = (isK ? k8 : q8) + ((int64_t)bh * ntiles * kTile + l0) * D;
#pragma unroll
    for (int i = tid; i < kTile * (D / 16); i += kTile) {
        const int r = i / (D / 16), c = i % (D / 16);
        reinterpret_cast<uint4*>(dst)[i] = *reinterpret_cast<const uint4*>(ost + r * OPITCH + 16 * c);
    }
}

// ---------------------------------------------------------------- V e4m3
// One CTA of 128 threads per (b, h, 128-token tile). Thread t covers the
// channel pair (2p, 2p + 1), p = t % (D/2), over the token group t / (D/2).
// Writes V transposed: v8t[b, h, d, token].
template <int D>
__global__ void __launch_bounds__(kTile) v_quant_kernel(View4 x, const float* __restrict__ vmul,
                                                        uint8_t* __restrict__ v8t, int vec) {
    constexpr int PITCH = D + 8;
    constexpr int P = D / 2;                     // channel pairs
    constexpr int G = kTile / P;                 // token groups
    constexpr int TT = kTile / G;                // tokens per thread
    constexpr int OPITCH = kTile + 16;           // staged output row pitch (bytes)
    static_assert(D * OPITCH <= kTile * PITCH * 2, "output staging reuses the tile");
    __shared__ __align__(128) uint16_t tile[kTile * PITCH];
    __shared__ float rmul[D];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;

    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    const int ntiles = static_cast<int>(ceil_div(L, kTile));
    const int bh = blockIdx.x / ntiles, tl = blockIdx.x % ntiles;
    const int b = bh / Hh, h = bh % Hh;
    const int tid = threadIdx.x;
    const int l0 = tl * kTile;
    const int nrows = min(kTile, L - l0);

    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (tid < D) rmul[tid] = vmul[(int64_t)bh * D + tid];
    __syncthreads();
    if (!stage_tile<D>(x, b, h, l0, nrows, vec != 0, tile, &bar, &abort_flag, 2)) return;

    const int p = tid % P, g = tid / P;
    const float r0 = rmul[2 * p], r1 = rmul[2 * p + 1];
    uint32_t w0[TT / 4], w1[TT / 4];
#pragma unroll
    for (int t4 = 0; t4 < TT / 4; ++t4) {
        float y0[4], y1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int tok = g * TT + 4 * t4 + i;
            const uint32_t u =
                tok < nrows ? *reinterpret_cast<const uint32_t*>(tile + tok * PITCH + 2 * p) : 0u;
            y0[i] = __fmul_rn(bf16_bits_to_f32(u & 0xFFFFu), r0);
            y1[i] = __fmul_rn(__uint_as_float(u & 0xFFFF0000u), r1);
        }
        w0[t4] = e4m3x2_rn_satfinite(y0[0], y0[1]) | (uint32_t(e4m3x2_rn_satfinite(y0[2], y0[3])) << 16);
        w1[t4] = e4m3x2_rn_satfinite(y1[0], y1[1]) | (uint32_t(e4m3x2_rn_satfinite(y1[2], y1[3])) << 16);
    }
    __syncthreads();              // every read of the tile is done
    uint8_t* ost = reinterpret_cast<uint8_t*>(tile);
#pragma unroll
    for (int c = 0; c < TT / 16; ++c) {
        *reinterpret_cast<uint4*>(ost + (2 * p) * OPITCH + g * TT + 16 * c) =
            make_uint4(w0[4 * c], w0[4 * c + 1], w0[4 * c + 2], w0[4 * c + 3]);
        *reinterpret_cast<uint4*>(ost + (2 * p + 1) * OPITCH + g * TT + 16 * c) =
            make_uint4(w1[4 * c], w1[4 * c + 1], w1[4 * c + 2], w1[4 * c + 3]);
    }
    __syncthreads();
    const int64_t Lpad = (int64_t)ntiles * kTile;
    uint8_t* dst = v8t + (int64_t)bh * D * Lpad + l0;
#pragma unroll
    for (int i = tid; i < D * (kTile / 16); i += kTile) {
        const int d = i / (kTile / 16), c = i % (kTile / 16);
        *reinterpret_cast<uint4*>(dst + (int64_t)d * Lpad + 16 * c) =
            *reinterpret_cast<const uint4*>(ost + d * OPITCH + 16 * c);
    }
}

}  // namespace

size_t quant_qk_ws_bytes(int B, int Hk, int Lk, int D) {
    (void)Lk;
    return (size_t)B * Hk * D * sizeof(float);
}

size_t quant_v_ws_bytes(int B, int Hk, int L, int D) {
    (void)L;
    return (size_t)B * Hk * D * sizeof(float);
}

cudaError_t launch_quant_qk(const View4& q, const View4& k, int blk_q, int blk_k, int8_t* q8,
                            float* q_scale, int8_t* k8, float* k_scale, float* k_mean, void* ws,
                            cudaStream_t s) {
    const int B = (int)q.size[0], H = (int)q.size[1], Lq = (int)q.size[2], D = (int)q.size[3];
    const int Hk = (int)k.size[1], Lk = (int)k.size[2];
    const int kvec = view_vec8(k), qvec = view_vec8(q);
    float* mean = static_cast<float*>(ws);
    const int sgrid = kStatCluster * B * Hk;
    const int n_qtiles = B * H * (int)ceil_div(Lq, kTile);
    const int n_ktiles = B * Hk * (int)ceil_div(Lk, kTile);
    if (D == 128) {
        column_stats_kernel<128, 0><<<sgrid, kStatThreads, 0, s>>>(k, mean, k_mean, kvec);
        qk_quant_kernel<128><<<n_qtiles + n_ktiles, kTile, 0, s>>>(
            q, k, blk_q, blk_k, n_qtiles, mean, q8, q_scale, k8, k_scale, qvec, kvec);
    } else {
        column_stats_kernel<64, 0><<<sgrid, kStatThreads, 0, s>>>(k, mean, k_mean, kvec);
        qk_quant_kernel<64><<<n_qtiles + n_ktiles, kTile, 0, s>>>(
            q, k, blk_q, blk_k, n_qtiles, mean, q8, q_scale, k8, k_scale, qvec, kvec);
    }
    return cudaGetLastError();
}

cudaError_t launch_quant_v(const View4& v, uint8_t* v8t, float* v_scale, void* ws,
                           cudaStream_t s) {
    const int B = (int)v.size[0], Hk = (int)v.size[1], L = (int)v.size[2], D = (int)v.size[3];
    const int vec = view_vec8(v);
    float* vmul = static_cast<float*>(ws);
    const int sgrid = kStatCluster * B * Hk;
    const int ntiles = B * Hk * (int)ceil_div(L, kTile);
    if (D == 128) {
        column_stats_kernel<128, 1><<<sgrid, kStatThreads, 0, s>>>(v, vmul, v_scale, vec);
        v_quant_kernel<128><<<ntiles, kTile, 0, s>>>(v, vmul, v8t, vec);
    } else {
        column_stats_kernel<64, 1><<<sgrid, kStatThreads, 0, s>>>(v, vmul, v_scale, vec);
        v_quant_kernel<64><<<ntiles, kTile, 0, s>>>(v, vmul, v8t, vec);
    }
    return cudaGetLastError();
}

unsigned read_clear_quant_error() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_quant_err, sizeof v) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_quant_err, &zero, sizeof zero);
    return v;
}

}  // namespace sage

// ---------------------------------------------------------------- no-allocation variant
// sage_quant_qk_noalloc: the same Q/K smoothing + rotation + INT8 quantisation
// as sage_quant_qk, for callers that cannot allocate device memory at the
// point of the call -- for instance a serving loop whose device memory is
// budgeted once at start-up, or code that must not risk the implicit device
// synchronisation that cudaMalloc / cudaFree can cause. Its scratch (the fp32
// per-channel mean of K, written by the statistics kernel before the
// quantisation kernel reads it) lives in the fixed array below instead of a
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
