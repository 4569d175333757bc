// quant.cu -- K smoothing statistics, fused smooth + Hadamard + INT8
// quantisation of Q and K, and FP8 e4m3 per-channel quantisation of V.
//
// Numerics are a fixed operation graph so that results are bit-identical
// to a plain sequential evaluation (this TU is compiled with -fmad=false,
// and every rounding step uses an explicit _rn intrinsic):
//   mean_K = fp32(fp64 sum / L)           (fp64 partial sums per CTA, per
//                                          cluster, then clusters in order)
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
// Kernels:
//   column_stats_kernel  clusters of 8 CTAs, `parts` clusters per (b, h),
//                        each streaming a contiguous token range; a
//                        cluster's CTAs reduce through distributed shared
//                        memory and its leader writes the partial column
//                        statistic (fp64 sums for K, fp32 maxima for V).
//   qk_quant_kernel      persistent CTAs over 128-token tiles (Q tiles, then
//                        K tiles), launched as a programmatic dependent of
//                        the K statistics kernel: Q tiles run while the
//                        statistics are computed, K tiles wait for them. Each CTA keeps two tiles in flight: the
//                        next tile arrives in shared memory by coalesced
//                        16-byte cp.async copies while the current one is
//                        converted, one
//                        thread per token row, all log2(D) butterfly stages
//                        inside the thread (f32x2 pairs), codes stored
//                        straight from registers.
//   v_quant_kernel       the same ring; output written transposed
//                        [b, h, d, token].
#include <algorithm>
#include <type_traits>

#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"
#include "quant_rows.cuh"

namespace sage {

__device__ unsigned g_quant_err;

namespace {

using namespace qrow;
namespace cg = cooperative_groups;

constexpr int kStatCluster = 8;      // CTAs per cluster in the statistics kernel
constexpr int kStatThreads = 256;
constexpr int kStatUnroll = 8;       // 16-byte loads in flight per thread
constexpr int kMaxParts = 8;         // clusters per (b, h), at most
constexpr int kQuantCtasPerSm = 3;   // resident quantisation CTAs per SM

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
// grid (8 * parts * B*Hh), 256 threads, clusters of 8 along x. Cluster c =
// blockIdx.x / 8 covers head bh = c / parts, part c % parts; CTA `rank` of
// it covers tokens [(part * 8 + rank) * span, + span).
// MODE 0 (K): fp64 column sums -> ws[(bh * parts + part) * D + d] (double).
// MODE 1 (V): fp32 column absmax -> ws[(bh * parts + part) * D + d] (float).
template <int D, int MODE>
__global__ void __cluster_dims__(kStatCluster, 1, 1) __launch_bounds__(kStatThreads)
    column_stats_kernel(View4 x, int parts, void* __restrict__ ws, int vec) {
    pdl_launch_dependents();                      // the quantisation kernel may start now
    constexpr int TPR = D / 8;                    // threads per token row
    constexpr int RPI = kStatThreads / TPR;       // token rows per load round
    using Acc = typename std::conditional<MODE == 0, double, float>::type;
    __shared__ Acc red[RPI][D];
    __shared__ Acc part_s[D];

    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    const int rank = blockIdx.x % kStatCluster;
    const int cid = blockIdx.x / kStatCluster;
    const int bh = cid / parts, part = cid % parts;
    const int b = bh / Hh, h = bh % Hh;
    const int tid = threadIdx.x;
    const int cg8 = tid % TPR, rg = tid / TPR;
    const int span = static_cast<int>(ceil_div(L, kStatCluster * parts));
    const int l0 = (part * kStatCluster + rank) * span;
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
        part_s[tid] = s;
    }
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();
    if (rank == 0 && tid < D) {
        Acc s = part_s[tid];
        for (int r = 1; r < kStatCluster; ++r) {
            const Acc o = cl.map_shared_rank(part_s, r)[tid];
            if (MODE == 0) s = __dadd_rn(s, o);
            else s = fmaxf(s, o);
        }
        static_cast<Acc*>(ws)[((int64_t)bh * parts + part) * D + tid] = s;
    }
    cl.sync();                  // the leader has read every CTA's partials
}

// ---------------------------------------------------------------- staging
// Shared-memory image of one 128-token tile: row r at r * (D + 8) elements
// (rows land 16 bytes apart in the bank space, so a thread reading its own
// row conflicts with nobody).
template <int D>
struct Tile {
    static constexpr int kPitch = D + 8;
    static constexpr int kElems = kTile * kPitch;
};

// Start bringing rows [0, nrows) of a 128-token tile of head (b, h) into
// `tile`: the CTA's 128 threads issue 16-byte asynchronous copies
// (cp.async, consecutive threads on consecutive 16 bytes of a row) and
// commit them as one group. Only for views whose rows are contiguous and
// 16-byte aligned.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
__device__ __forceinline__ void issue_tile(const View4& x, int b, int h, int l0, int nrows,
                                           uint16_t* tile) {
    constexpr int CPR = D / 8;                     // 16-byte chunks per row
    const uint16_t* base = static_cast<const uint16_t*>(x.ptr);
    const int64_t hoff = b * x.stride[0] + h * x.stride[1];
    for (int i = threadIdx.x; i < nrows * CPR; i += kTile) {
        const int r = i / CPR, c = i % CPR;
        cp_async16(tile + r * Tile<D>::kPitch + 8 * c, base + hoff + (int64_t)(l0 + r) * x.stride[2] + 8 * c);
    }
}

// Strided element gather of the same rows by the whole CTA (any view).
template <int D>
__device__ __forceinline__ void gather_tile(const View4& x, int b, int h, int l0, int nrows,
                                            uint16_t* tile) {
    const uint16_t* base = static_cast<const uint16_t*>(x.ptr);
    const int64_t hoff = b * x.stride[0] + h * x.stride[1];
    for (int i = threadIdx.x; i < nrows * D; i += kTile) {
        const int r = i / D, d = i % D;
        tile[r * Tile<D>::kPitch + d] =
            __ldg(base + hoff + (int64_t)(l0 + r) * x.stride[2] + (int64_t)d * x.stride[3]);
    }
}

// One 128-token tile of the Q-then-K tile list: tiles [0, n_qtiles) walk Q
// head by head, the rest walk K.
struct QkTile {
    bool isK;
    int bh, b, h, tl, l0, nrows, ntiles;
};

__device__ __forceinline__ QkTile qk_tile(int t, int n_qtiles, const View4& q, const View4& k) {
    QkTile r;
    r.isK = t >= n_qtiles;
    const View4& x = r.isK ? k : q;
    const int lin = r.isK ? t - n_qtiles : t;
    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    r.ntiles = static_cast<int>(ceil_div(L, kTile));
    r.bh = lin / r.ntiles;
    r.tl = lin % r.ntiles;
    r.b = r.bh / Hh;
    r.h = r.bh % Hh;
    r.l0 = r.tl * kTile;
    r.nrows = min(kTile, L - r.l0);
    return r;
}

// ---------------------------------------------------------------- Q/K int8
// Persistent CTAs of 128 threads; CTA c takes tiles c, c + G, c + 2G, ...
// (G = gridDim.x) and thread r owns token row r of the current tile. Two
// shared-memory tile buffers alternate: while tile i is converted, tile
// i + 1 is in flight. The K mean of a head is finished here from the
// statistics kernel's per-cluster fp64 sums (in cluster order).
template <int D>
__global__ void __launch_bounds__(kTile) qk_quant_kernel(
    View4 q, View4 k, int blk_q, int blk_k, int n_qtiles, int n_tiles,
    const double* __restrict__ ksum, int parts, int8_t* __restrict__ q8,
    float* __restrict__ q_scale, int8_t* __restrict__ k8, float* __restrict__ k_scale,
    float* __restrict__ k_mean, int qvec, int kvec) {
    constexpr int PITCH = Tile<D>::kPitch;        // staged input row pitch (elements)
    extern __shared__ __align__(128) uint16_t qk_smem[];
    uint16_t* tiles = qk_smem;                    // [2][Tile<D>::kElems]
    __shared__ __align__(16) float mean_s[D];
    __shared__ float wmax[kTile / 32];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    auto is_vec = [&](const QkTile& tr) { return (tr.isK ? kvec : qvec) != 0; };
    // every thread commits one copy group per tile slot (empty for gathered
    // tiles), so "at most one group pending" always means "the current tile
    // has landed"
    auto start = [&](int t, int buf) {
        if (t < n_tiles) {
            const QkTile tr = qk_tile(t, n_qtiles, q, k);
            if (is_vec(tr))
                issue_tile<D>(tr.isK ? k : q, tr.b, tr.h, tr.l0, tr.nrows, tiles + buf * Tile<D>::kElems);
        }
        cp_async_commit();
    };
    const int G = gridDim.x;
    start(blockIdx.x, 0);
    start(blockIdx.x + G, 1);

    bool stats_ready = false;
    for (int it = 0, t = blockIdx.x; t < n_tiles; ++it, t += G) {
        const int buf = it & 1;
        uint16_t* tile = tiles + buf * Tile<D>::kElems;
        const QkTile tr = qk_tile(t, n_qtiles, q, k);
        const View4& x = tr.isK ? k : q;
        if (tr.isK && !stats_ready) {
            // Q tiles ran alongside the statistics kernel; K tiles need its sums
            pdl_wait();
            stats_ready = true;
        }
        if (tr.isK && tid < D) {
            double sum = 0.0;
            for (int pp = 0; pp < parts; ++pp) sum = __dadd_rn(sum, ksum[((int64_t)tr.bh * parts + pp) * D + tid]);
            const float mn = __double2float_rn(__ddiv_rn(sum, (double)x.size[2]));
            mean_s[tid] = mn;
            if (k_mean != nullptr && tr.tl == 0) k_mean[(int64_t)tr.bh * D + tid] = mn;
        }
        cp_async_wait<1>();                      // this thread's copies of tile t are in
        if (!is_vec(tr)) gather_tile<D>(x, tr.b, tr.h, tr.l0, tr.nrows, tile);
        __syncthreads();                         // everyone's copies (and mean_s) are in

        const bool valid = tid < tr.nrows;
        uint64_t x2[D / 2];
        {
            const uint16_t* row = tile + tid * PITCH;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 u = valid ? *reinterpret_cast<const uint4*>(row + 8 * c) : make_uint4(0, 0, 0, 0);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    x2[4 * c + e] = p2(bf16_bits_to_f32(w[e] & 0xFFFFu), __uint_as_float(w[e] & 0xFFFF0000u));
            }
        }
        if (tr.isK && valid) {
#pragma unroll
            for (int c = 0; c < D / 2; ++c) x2[c] = p2sub(x2[c], *reinterpret_cast<const uint64_t*>(mean_s + 2 * c));
        }
        butterfly_pairs<D>(x2);

        float a = 0.0f;
#pragma unroll
        for (int j = 0; j < D / 2; ++j) a = fmax3(a, fabsf(p2lo(x2[j])), fabsf(p2hi(x2[j])));
        // a >= +0, so the bit patterns order like the values
        const unsigned am = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
        if (lane == 0) wmax[warp] = __uint_as_float(am);
        __syncthreads();              // every row has left the buffer; block maxima are in
        start(t + 2 * G, buf);
        const int blk = tr.isK ? blk_k : blk_q;
        const int nb = static_cast<int>(ceil_div(x.size[2], blk));
        const int wpb = blk / 32;     // warps per quantisation block (blk in {32, 64, 128})
        const int w0 = (warp / wpb) * wpb;
        float amax = 0.0f;
        for (int w = w0; w < w0 + wpb; ++w) amax = fmaxf(amax, wmax[w]);
        float s = 0.0f, rr = 0.0f;
        if (amax != 0.0f) {
            s = __fdiv_rn(amax, 127.0f);
            rr = __fdiv_rn(127.0f, amax);
        }
        const int l = tr.l0 + tid;
        if (valid && (l & (blk - 1)) == 0) {
            float* scales = tr.isK ? k_scale : q_scale;
            scales[(int64_t)tr.bh * nb + l / blk] = s;
        }

        // Each thread stores its own code row (rows past L are the zero
        // padding).
        uint4* dst = reinterpret_cast<uint4*>((tr.isK ? k8 : q8) +
                                              ((int64_t)tr.bh * tr.ntiles * kTile + tr.l0 + tid) * D);
#pragma unroll
        for (int c = 0; c < D / 16; ++c) dst[c] = row_codes16<D>(x2, rr, c);
    }
}

// ---------------------------------------------------------------- V e4m3
// Persistent CTAs of 128 threads over 128-token tiles of V, the same
// two-buffer ring as qk_quant_kernel. Thread t covers the channel pair
// (2p, 2p + 1), p = t % (D/2), over the token group t / (D/2), and stores its
// codes straight to the transposed output v8t[b, h, d, token]. The channel
// maxima are finished here from the statistics kernel's per-cluster maxima;
// the first tile of each head also writes its v_scale.
template <int D>
__global__ void __launch_bounds__(kTile) v_quant_kernel(View4 x, int n_tiles,
                                                        const float* __restrict__ vmax, int parts,
                                                        float* __restrict__ v_scale,
                                                        uint8_t* __restrict__ v8t, int vec) {
    constexpr int PITCH = Tile<D>::kPitch;
    constexpr int P = D / 2;                     // channel pairs
    constexpr int G = kTile / P;                 // token groups
    constexpr int TT = kTile / G;                // tokens per thread
    extern __shared__ __align__(128) uint16_t v_smem[];
    uint16_t* tiles = v_smem;                    // [2][Tile<D>::kElems]
    __shared__ float rmul[D];

    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    const int ntiles = static_cast<int>(ceil_div(L, kTile));
    const int tid = threadIdx.x;

    // one copy group per tile slot and thread (empty for gathered views)
    auto start = [&](int t, int buf) {
        if (t < n_tiles && vec) {
            const int bh = t / ntiles, tl = t % ntiles;
            issue_tile<D>(x, bh / Hh, bh % Hh, tl * kTile, min(kTile, L - tl * kTile),
                          tiles + buf * Tile<D>::kElems);
        }
        cp_async_commit();
    };
    const int GS = gridDim.x;
    start(blockIdx.x, 0);
    start(blockIdx.x + GS, 1);
    pdl_wait();                                  // the channel maxima are complete
    pdl_launch_dependents();                     // the attention kernel may start its prologue

    const int p = tid % P, g = tid / P;
    for (int it = 0, t = blockIdx.x; t < n_tiles; ++it, t += GS) {
        const int buf = it & 1;
        uint16_t* tile = tiles + buf * Tile<D>::kElems;
        const int bh = t / ntiles, tl = t % ntiles;
        const int l0 = tl * kTile;
        const int nrows = min(kTile, L - l0);
        if (tid < D) {
            float a = 0.0f;
            for (int pp = 0; pp < parts; ++pp) a = fmaxf(a, vmax[((int64_t)bh * parts + pp) * D + tid]);
            float sc = 0.0f, r = 0.0f;
            if (a != 0.0f) {
                sc = __fdiv_rn(a, 448.0f);
                r = __fdiv_rn(448.0f, a);
            }
            rmul[tid] = r;
            if (tl == 0) v_scale[(int64_t)bh * D + tid] = sc;
        }
        cp_async_wait<1>();                      // this thread's copies of tile t are in
        if (!vec) gather_tile<D>(x, bh / Hh, bh % Hh, l0, nrows, tile);
        __syncthreads();                         // everyone's copies (and rmul) are in

        const uint64_t r2 = p2(rmul[2 * p], rmul[2 * p + 1]);
        uint32_t w0[TT / 4], w1[TT / 4];
#pragma unroll
        for (int t4 = 0; t4 < TT / 4; ++t4) {
            float y0[4], y1[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tok = g * TT + 4 * t4 + i;
                const uint32_t u =
                    tok < nrows ? *reinterpret_cast<const uint32_t*>(tile + tok * PITCH + 2 * p) : 0u;
                const uint64_t y = p2mul(p2(bf16_bits_to_f32(u & 0xFFFFu), __uint_as_float(u & 0xFFFF0000u)), r2);
                y0[i] = p2lo(y);
                y1[i] = p2hi(y);
            }
            w0[t4] = e4m3x2_rn_satfinite(y0[0], y0[1]) | (uint32_t(e4m3x2_rn_satfinite(y0[2], y0[3])) << 16);
            w1[t4] = e4m3x2_rn_satfinite(y1[0], y1[1]) | (uint32_t(e4m3x2_rn_satfinite(y1[2], y1[3])) << 16);
        }
        __syncthreads();              // every read of the buffer is done
        start(t + 2 * GS, buf);
        // channels 2p and 2p + 1, tokens [g TT, g TT + TT) of the tile: two
        // contiguous runs of TT bytes in the transposed output
        const int64_t Lpad = (int64_t)ntiles * kTile;
        uint8_t* dst = v8t + ((int64_t)bh * D + 2 * p) * Lpad + l0 + g * TT;
#pragma unroll
        for (int c = 0; c < TT / 16; ++c) {
            reinterpret_cast<uint4*>(dst)[c] = make_uint4(w0[4 * c], w0[4 * c + 1], w0[4 * c + 2], w0[4 * c + 3]);
            reinterpret_cast<uint4*>(dst + Lpad)[c] =
                make_uint4(w1[4 * c], w1[4 * c + 1], w1[4 * c + 2], w1[4 * c + 3]);
        }
    }
}

// Clusters per (b, h) for the statistics kernels: about three 256-thread
// CTAs per SM over the whole grid, between 1 and kMaxParts.
int stat_parts(int BH) {
    const int want = num_sms() * 3;
    const int per_part = BH * kStatCluster;
    return std::max(1, std::min(kMaxParts, (want + per_part / 2) / per_part));
}

template <int D>
size_t quant_smem_bytes() {
    return 2 * Tile<D>::kElems * sizeof(uint16_t);
}

template <int D>
cudaError_t launch_qk_d(const View4& q, const View4& k, int blk_q, int blk_k, int8_t* q8,
                        float* q_scale, int8_t* k8, float* k_scale, float* k_mean, void* ws,
                        cudaStream_t s, bool with_q) {
    const int B = (int)q.size[0], H = (int)q.size[1], Lq = (int)q.size[2];
    const int Hk = (int)k.size[1], Lk = (int)k.size[2];
    const int parts = stat_parts(B * Hk);
    column_stats_kernel<D, 0><<<kStatCluster * parts * B * Hk, kStatThreads, 0, s>>>(
        k, parts, ws, view_vec8(k));
    const int n_qtiles = with_q ? B * H * (int)ceil_div(Lq, kTile) : 0;
    const int n_tiles = n_qtiles + B * Hk * (int)ceil_div(Lk, kTile);
    const int grid = std::min(n_tiles, num_sms() * kQuantCtasPerSm);
    auto kern = qk_quant_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)quant_smem_bytes<D>());
    if (e != cudaSuccess) return e;
    // programmatic launch: the Q tiles overlap the statistics kernel
    e = launch_pdl(kern, dim3(grid), dim3(kTile), quant_smem_bytes<D>(), s, q, k, blk_q, blk_k,
                   n_qtiles, n_tiles, static_cast<const double*>(ws), parts, q8, q_scale, k8,
                   k_scale, k_mean, view_vec8(q), view_vec8(k));
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D>
cudaError_t launch_v_d(const View4& v, uint8_t* v8t, float* v_scale, void* ws, cudaStream_t s) {
    const int B = (int)v.size[0], Hk = (int)v.size[1], L = (int)v.size[2];
    const int parts = stat_parts(B * Hk);
    column_stats_kernel<D, 1><<<kStatCluster * parts * B * Hk, kStatThreads, 0, s>>>(
        v, parts, ws, view_vec8(v));
    const int n_tiles = B * Hk * (int)ceil_div(L, kTile);
    const int grid = std::min(n_tiles, num_sms() * kQuantCtasPerSm);
    auto kern = v_quant_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)quant_smem_bytes<D>());
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(grid), dim3(kTile), quant_smem_bytes<D>(), s, v, n_tiles,
                   static_cast<const float*>(ws), parts, v_scale, v8t, view_vec8(v));
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

size_t quant_qk_ws_bytes(int B, int Hk, int Lk, int D) {
    (void)Lk;
    return (size_t)B * Hk * kMaxParts * D * sizeof(double);
}

size_t quant_v_ws_bytes(int B, int Hk, int L, int D) {
    (void)L;
    return (size_t)B * Hk * kMaxParts * D * sizeof(float);
}

cudaError_t launch_quant_qk(const View4& q, const View4& k, int blk_q, int blk_k, int8_t* q8,
                            float* q_scale, int8_t* k8, float* k_scale, float* k_mean, void* ws,
                            cudaStream_t s, bool with_q) {
    return k.size[3] == 128
               ? launch_qk_d<128>(q, k, blk_q, blk_k, q8, q_scale, k8, k_scale, k_mean, ws, s, with_q)
               : launch_qk_d<64>(q, k, blk_q, blk_k, q8, q_scale, k8, k_scale, k_mean, ws, s, with_q);
}

cudaError_t launch_quant_v(const View4& v, uint8_t* v8t, float* v_scale, void* ws,
                           cudaStream_t s) {
    return v.size[3] == 128 ? launch_v_d<128>(v, v8t, v_scale, ws, s)
                            : launch_v_d<64>(v, v8t, v_scale, ws, s);
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
// synchronisation that cudaMalloc / cudaFree can cause. Its scratch (the fp64
// per-cluster column sums of K, written by the statistics kernel before the
// quantisation kernel reads them) lives in the fixed array below instead of
// a caller workspace.
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
