// quant.cu -- K smoothing statistics, fused smooth + Hadamard + INT8
// quantisation of Q and K, and FP8 e4m3 per-channel quantisation of V.
//
// Numerics are a fixed operation graph so that results are bit-identical
// to a plain sequential evaluation (this TU is compiled with -fmad=false,
// and every rounding step uses an explicit _rn intrinsic):
//   mean_K = fp32(fp64 sum / L)           (fp64 sums of bf16 values, exact in
//                                          any order unless the magnitudes
//                                          span more than ~45 binades)
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
// Every call is two launches on the caller's stream:
//   head_stats_kernel    one cluster of 8 CTAs per (tensor, b, h). The CTAs
//                        stream contiguous eighths of the head's tokens
//                        through a four-stage cp.async ring and reduce
//                        through distributed shared memory; the leader
//                        writes the head's final statistic: the fp32
//                        K mean (workspace, and k_mean when asked), or for V
//                        the scale a / 448 (v_scale) and the multiplier
//                        448 / a (workspace).
//   quant_tiles_kernel   persistent 512-thread CTAs over one list of
//                        128-token tiles, launched as a programmatic
//                        dependent of the statistics: Q tiles first (they
//                        need no statistics), then K and V tiles alternating,
//                        so each SM mixes the butterfly-heavy K work with
//                        the copy-bound V work (tiles of a [B, L, H, D]
//                        view go heads fastest, so CTAs that run together
//                        read whole token rows). A CTA keeps three tiles in
//                        flight: 16-byte cp.async copies into a swizzled
//                        shared-memory ring, the head's statistic vector in
//                        the same copy group. Q and K: four threads per token
//                        row; the butterfly stages whose partner element sits
//                        in another thread of the quad exchange values by
//                        shuffle. V: one thread per channel pair and group of
//                        tokens, codes stored straight into the transposed
//                        output.
#include <algorithm>
#include <type_traits>

#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"
#include "quant_rows.cuh"

namespace sage {

namespace {

using namespace qrow;
namespace cg = cooperative_groups;

constexpr int kStatCluster = 8;      // CTAs per (tensor, head) in the statistics kernel
constexpr int kStatThreads = 256;
constexpr int kQThreads = 512;       // quantisation CTA: four threads per token row
constexpr int kQStages = 3;          // tiles in flight per quantisation CTA
constexpr int kQMinCtas = 2;         // resident quantisation CTAs per SM the kernel is built for

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

// ---------------------------------------------------------------- stats
// What one statistics launch covers: the nk heads (b, h) of K, then the nv
// heads of V, a cluster each.
struct StatsJob {
    View4 k, v;
    int nk, nv;
    int kvec, vvec;
    float* k_mean_ws;   // [nk][D] fp32 K mean (workspace)
    float* k_mean;      // [nk][D] caller's copy of the mean, or null
    float* v_rmul_ws;   // [nv][D] fp32 448 / a (0 for a = 0), workspace
    float* v_scale;     // [nv][D] a / 448
};

constexpr int kStatRows = 64;        // token rows per ring stage
constexpr int kStatStages = 4;       // ring stages in flight per CTA

template <int D>
constexpr size_t stat_smem_bytes() {
    return (size_t)kStatStages * kStatRows * D * sizeof(uint16_t);
}

// One CTA's share of head `bh`: tokens [rank * span, + span), span =
// ceil(L / 8), streamed through a ring of kStatStages stages of 64 token
// rows (16-byte cp.async; a strided view is gathered with plain loads
// instead). Thread t accumulates the column pair cp = t % (D / 2) over its
// group of rows of every stage. MODE 0 (K): fp64 sums, finished into the
// fp32 mean. MODE 1 (V): the absmax of the bf16 values (|x| and max are exact
// in bf16), finished into scale and multiplier.
template <int D, int MODE>
__device__ __forceinline__ void head_stats(const View4& x, int bh, int rank, int vec,
                                           unsigned char* smem, float* ws_out, float* out2) {
    constexpr int CPR = D / 8;                    // 16-byte chunks per token row
    constexpr int RPP = kStatThreads / CPR;       // rows one pass of copies covers
    constexpr int NPASS = kStatRows / RPP;        // copy passes per stage
    constexpr int NCP = D / 2;                    // column pairs
    constexpr int NRG = kStatThreads / NCP;       // row groups
    constexpr int RPG = kStatRows / NRG;          // rows of a stage per group
    constexpr int kStageElems = kStatRows * D;
    using Acc = typename std::conditional<MODE == 0, double, float>::type;
    uint16_t* ring = reinterpret_cast<uint16_t*>(smem);

    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    const int b = bh / Hh, h = bh % Hh;
    const int tid = threadIdx.x;
    const int span = static_cast<int>(ceil_div(L, kStatCluster));
    const int l0 = min(L, rank * span);
    const int l1 = min(L, l0 + span);
    const int nst = static_cast<int>(ceil_div(l1 - l0, kStatRows));
    const int64_t rs = x.stride[2];
    const uint16_t* hbase = static_cast<const uint16_t*>(x.ptr) + b * x.stride[0] + h * x.stride[1];
    const int cr = tid / CPR, cc = tid % CPR;

    // one copy group per stage slot and thread (empty past the end and for
    // gathered views)
    auto issue = [&](int st) {
        if (st < nst && vec) {
            const int r0 = l0 + st * kStatRows;
            const int nr = min(kStatRows, l1 - r0);
            uint16_t* dst = ring + (st % kStatStages) * kStageElems + cr * D + 8 * cc;
            const uint16_t* src = hbase + (int64_t)(r0 + cr) * rs + 8 * cc;
#pragma unroll
            for (int k = 0; k < NPASS; ++k)
                if (cr + k * RPP < nr) cp_async16(dst + k * RPP * D, src + (int64_t)(k * RPP) * rs);
        }
        cp_async_commit();
    };
#pragma unroll
    for (int st = 0; st < kStatStages; ++st) issue(st);

    const int cp = tid % NCP, rg = tid / NCP;
    double s0 = 0.0, s1 = 0.0;                    // MODE 0: columns 2cp, 2cp + 1
    __nv_bfloat162 mx = __floats2bfloat162_rn(0.0f, 0.0f);   // MODE 1
    for (int st = 0; st < nst; ++st) {
        const int r0 = l0 + st * kStatRows;
        const int nr = min(kStatRows, l1 - r0);
        uint16_t* stage = ring + (st % kStatStages) * kStageElems;
        cp_async_wait<kStatStages - 1>();         // this thread's copies of the stage are in
        if (!vec) {
            for (int i = tid; i < nr * D; i += kStatThreads) {
                const int r = i / D, d = i % D;
                stage[r * D + d] = __ldg(hbase + (int64_t)(r0 + r) * rs + (int64_t)d * x.stride[3]);
            }
        }
        __syncthreads();                          // everyone's copies are in
        const uint32_t* col = reinterpret_cast<const uint32_t*>(stage + rg * RPG * D) + cp;
#pragma unroll
        for (int i = 0; i < RPG; ++i) {
            uint32_t u = col[i * (D / 2)];
            if (rg * RPG + i >= nr) u = 0u;       // rows past the CTA's range
            if (MODE == 0) {
                s0 = __dadd_rn(s0, (double)bf16_bits_to_f32(u & 0xFFFFu));
                s1 = __dadd_rn(s1, (double)__uint_as_float(u & 0xFFFF0000u));
            } else {
                mx = __hmax2(mx, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&u)));
            }
        }
        __syncthreads();                          // the stage has been read
        issue(st + kStatStages);
    }

    // the ring is idle now (every later copy group is empty): reduce the row
    // groups through it, then the cluster's CTAs through distributed shared
    // memory
    Acc* red = reinterpret_cast<Acc*>(smem);      // [NRG][D]
    Acc* part_s = red + NRG * D;                  // [D]
    if (MODE == 0) {
        red[rg * D + 2 * cp] = s0;
        red[rg * D + 2 * cp + 1] = s1;
    } else {
        const float2 f = __bfloat1622float2(mx);
        red[rg * D + 2 * cp] = f.x;
        red[rg * D + 2 * cp + 1] = f.y;
    }
    __syncthreads();
    if (tid < D) {
        Acc s = red[tid];
        for (int r = 1; r < NRG; ++r) {
            if (MODE == 0) s = __dadd_rn(s, red[r * D + tid]);
            else s = fmaxf(s, red[r * D + tid]);
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
        const int64_t o = (int64_t)bh * D + tid;
        if (MODE == 0) {
            const float mn = __double2float_rn(__ddiv_rn(s, (double)L));
            ws_out[o] = mn;
            if (out2 != nullptr) out2[o] = mn;
        } else {
            float sc = 0.0f, rm = 0.0f;
            if (s != 0.0f) {
                sc = __fdiv_rn(s, 448.0f);
                rm = __fdiv_rn(448.0f, s);
            }
            out2[o] = sc;
            ws_out[o] = rm;
        }
    }
    cl.sync();                  // the leader has read every CTA's partials
}

// grid 8 * (nk + nv), clusters of 8 along x: cluster c < nk covers K head c,
// the others V head c - nk.
template <int D>
__global__ void __cluster_dims__(kStatCluster, 1, 1) __launch_bounds__(kStatThreads)
    head_stats_kernel(StatsJob j) {
    pdl_launch_dependents();                      // the quantisation kernel may start now
    extern __shared__ __align__(128) unsigned char stat_smem[];
    const int rank = blockIdx.x % kStatCluster;
    const int c = blockIdx.x / kStatCluster;
    if (c < j.nk) head_stats<D, 0>(j.k, c, rank, j.kvec, stat_smem, j.k_mean_ws, j.k_mean);
    else head_stats<D, 1>(j.v, c - j.nk, rank, j.vvec, stat_smem, j.v_rmul_ws, j.v_scale);
}

// ---------------------------------------------------------------- staging
// Shared-memory image of one 128-token tile: row r at r * D elements, its
// 16-byte chunk c stored at chunk c ^ 4 (r & 1). Eight threads copying eight
// consecutive chunks of a row, a quad reading chunks 4m .. 4m + 3 of two
// neighbouring rows, or a warp reading 128 consecutive bytes of one row then
// touch eight distinct 16-byte bank groups.
__device__ __forceinline__ int swz(int r, int c) { return c ^ ((r & 1) << 2); }


// Strided element gather of the same rows by the whole CTA (any view).
template <int D>
__device__ __forceinline__ void gather_tile(const View4& x, int b, int h, int l0, int nrows,
                                            uint16_t* tile) {
    const uint16_t* base = static_cast<const uint16_t*>(x.ptr);
    const int64_t hoff = b * x.stride[0] + h * x.stride[1];
    for (int i = threadIdx.x; i < nrows * D; i += kQThreads) {
        const int r = i / D, d = i % D;
        tile[r * D + 8 * swz(r, d >> 3) + (d & 7)] =
            __ldg(base + hoff + (int64_t)(l0 + r) * x.stride[2] + (int64_t)d * x.stride[3]);
    }
}

// ---------------------------------------------------------------- tile list
struct QuantJob {
    View4 q, k, v;
    int nq, nk, nv;              // tiles of Q, K and V in the list
    int blk_q, blk_k;
    int qvec, kvec, vvec;
    const float* k_mean_ws;      // [B * Hk][D], written by the statistics kernel
    const float* v_rmul_ws;      // [B * Hk][D]
    int8_t* q8;
    float* q_scale;
    int8_t* k8;
    float* k_scale;
    uint8_t* v8t;
    // MXFP4 outputs (quant_tiles_kernel<D, true>): E2M1 codes and e8m0 scales
    uint8_t* q4;
    uint8_t* q_sf;
    uint8_t* k4;
    uint8_t* k_sf;
};

enum : int { kKindQ = 0, kKindK = 1, kKindV = 2 };

struct TileRef {
    int kind, bh, b, h, tl, l0, nrows, ntiles;
};

__device__ __forceinline__ const View4& view_of(const QuantJob& j, int kind) {
    return kind == kKindQ ? j.q : (kind == kKindK ? j.k : j.v);
}
__device__ __forceinline__ bool vec_of(const QuantJob& j, int kind) {
    return (kind == kKindQ ? j.qvec : (kind == kKindK ? j.kvec : j.vvec)) != 0;
}

// Tile t of the list: Q tiles [0, nq); then, when K and V are both present
// (nk == nv), K tile i at nq + 2i and V tile i at nq + 2i + 1; else the K or
// the V tiles in order. Within a tensor the tiles go head by head, or, when
// the view's heads lie closer in memory than its tokens (a [B, L, H, D]
// tensor), token range by token range with the heads fastest: the CTAs
// working at the same time then read whole contiguous token rows.
__device__ __forceinline__ TileRef tile_ref(int t, const QuantJob& j) {
    TileRef r;
    int lin;
    if (t < j.nq) {
        r.kind = kKindQ;
        lin = t;
    } else {
        const int u = t - j.nq;
        if (j.nk > 0 && j.nv > 0) {
            r.kind = (u & 1) ? kKindV : kKindK;
            lin = u >> 1;
        } else {
            r.kind = j.nk > 0 ? kKindK : kKindV;
            lin = u;
        }
    }
    const View4& x = view_of(j, r.kind);
    const int L = static_cast<int>(x.size[2]);
    const int Hh = static_cast<int>(x.size[1]);
    r.ntiles = static_cast<int>(ceil_div(L, kTile));
    if (x.stride[1] < x.stride[2]) {
        const int nbh = static_cast<int>(x.size[0]) * Hh;
        r.bh = lin % nbh;
        r.tl = lin / nbh;
    } else {
        r.bh = lin / r.ntiles;
        r.tl = lin % r.ntiles;
    }
    r.b = r.bh / Hh;
    r.h = r.bh % Hh;
    r.l0 = r.tl * kTile;
    r.nrows = min(kTile, L - r.l0);
    return r;
}

// Everything a CTA needs about one tile of the list, built once per tile by
// one thread (index arithmetic and 64-bit addresses stay off the other 511).
struct TileDesc {
    const uint16_t* src;   // element (row l0, d = 0) of the tile's head
    const float* stat;     // K: the head's mean; V: its multipliers 448 / a; Q: null
    void* out;             // Q/K: codes of row l0; V: v8t[b, h, 0, l0]
    float* scale;          // Q/K: scale of the block holding row l0
    uint8_t* sf;           // MXFP4 Q/K: the tile's 512-byte scale-factor block
    int64_t rstride;       // token-row stride of the view (elements)
    int64_t lpad;          // V: row pitch of the transposed output
    int kind, nrows, vec, blk;
    int b, h, l0, unused;
};

template <int D, bool MX>
__device__ TileDesc make_desc(int t, const QuantJob& j) {
    const TileRef r = tile_ref(t, j);
    const View4& x = view_of(j, r.kind);
    TileDesc d;
    d.kind = r.kind;
    d.nrows = r.nrows;
    d.vec = vec_of(j, r.kind) ? 1 : 0;
    d.b = r.b;
    d.h = r.h;
    d.l0 = r.l0;
    d.unused = 0;
    d.src = static_cast<const uint16_t*>(x.ptr) + r.b * x.stride[0] + r.h * x.stride[1] +
            (int64_t)r.l0 * x.stride[2];
    d.rstride = x.stride[2];
    d.lpad = (int64_t)r.ntiles * kTile;
    d.sf = nullptr;
    if (r.kind == kKindV) {
        d.blk = 0;
        d.stat = j.v_rmul_ws + (int64_t)r.bh * D;
        d.out = j.v8t + (int64_t)r.bh * D * d.lpad + r.l0;
        d.scale = nullptr;
    } else if (MX) {
        const bool isK = r.kind == kKindK;
        d.blk = 0;
        d.stat = isK ? j.k_mean_ws + (int64_t)r.bh * D : nullptr;
        d.out = (isK ? j.k4 : j.q4) + ((int64_t)r.bh * d.lpad + r.l0) * (D / 2);
        d.scale = nullptr;
        d.sf = (isK ? j.k_sf : j.q_sf) + ((int64_t)r.bh * d.lpad + r.l0) / kTile * 512;
    } else {
        const bool isK = r.kind == kKindK;
        d.blk = isK ? j.blk_k : j.blk_q;
        const int64_t nb = ceil_div(x.size[2], d.blk);
        d.stat = isK ? j.k_mean_ws + (int64_t)r.bh * D : nullptr;
        d.out = (isK ? j.k8 : j.q8) + ((int64_t)r.bh * d.lpad + r.l0) * D;
        d.scale = (isK ? j.k_scale : j.q_scale) + (int64_t)r.bh * nb + r.l0 / d.blk;
    }
    return d;
}

// ---------------------------------------------------------------- Q/K rows
// The butterfly of `butterfly` on a row spread over a quad of threads:
// thread `sub` holds elements j = 32 m + 8 sub + i (i = 0..7) as the pairs
// x2[4 m + i / 2]. Stages h = 1, 2, 4 and h >= 32 pair elements inside one
// thread; h = 8 and h = 16 pair thread sub with sub ^ 1 and sub ^ 2, whose
// values come by shuffle. In those two stages the thread holding x_j (bit
// clear) keeps x_j + x_{j+h} and its partner keeps x_j - x_{j+h}, each as
// fma(+-1, own value, partner's value): the product by +-1 is exact, so it
// is the same single rounding as the add or the subtract. Every stage is
// taken in ascending order with the same operands, so the bits equal the
// sequential butterfly's. Every lane must execute this (shuffles).
template <int D>
__device__ __forceinline__ void quad_butterfly(uint64_t (&x2)[D / 8], int sub) {
    constexpr int NP = D / 8;
#pragma unroll
    for (int k = 0; k < NP; ++k) {                       // h = 1
        const float a = p2lo(x2[k]), c = p2hi(x2[k]);
        x2[k] = p2(__fadd_rn(a, c), __fsub_rn(a, c));
    }
#pragma unroll
    for (int hp = 1; hp <= 2; hp <<= 1) {                // h = 2, 4
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            if (k & hp) continue;
            const uint64_t a = x2[k], c = x2[k + hp];
            x2[k] = p2add(a, c);
            x2[k + hp] = p2sub(a, c);
        }
    }
#pragma unroll
    for (int bit = 0; bit < 2; ++bit) {                  // h = 8, 16
        const float sg = ((sub >> bit) & 1) ? -1.0f : 1.0f;
        const uint64_t sg2 = p2(sg, sg);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const float ylo = __shfl_xor_sync(0xffffffffu, p2lo(x2[k]), 1 << bit);
            const float yhi = __shfl_xor_sync(0xffffffffu, p2hi(x2[k]), 1 << bit);
            x2[k] = p2fma(sg2, x2[k], p2(ylo, yhi));
        }
    }
#pragma unroll
    for (int hp = 4; hp < NP; hp <<= 1) {                // h = 32, 64
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            if (k & hp) continue;
            const uint64_t a = x2[k], c = x2[k + hp];
            x2[k] = p2add(a, c);
            x2[k + hp] = p2sub(a, c);
        }
    }
}

// Codes of the eight values held as pairs x2[k0 .. k0 + 3]: rne(x_hat * rr),
// four codes per word (value 2 k0 + 4i + e in byte e of word i), the same
// arithmetic as row_codes16. codes8_magic for a finite rr (|x_hat * rr| <=
// 127, so the magic-number rounding needs no clamp), codes8_clamp for the
// block whose 127 / a overflowed.
template <int N>
__device__ __forceinline__ uint2 codes8_magic(const uint64_t (&x2)[N], int k0, float rr) {
    const uint64_t rr2 = p2(rr, rr), mg2 = p2(kRoundMagic, kRoundMagic);
    uint32_t w[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        // the product is rounded on its own (an FMA with +0), so the magic
        // add that follows cannot be contracted into it
        const uint64_t t01 = p2add(p2fma(x2[k0 + 2 * i], rr2, 0ull), mg2);
        const uint64_t t23 = p2add(p2fma(x2[k0 + 2 * i + 1], rr2, 0ull), mg2);
        w[i] = __byte_perm(__byte_perm(__float_as_uint(p2lo(t01)), __float_as_uint(p2hi(t01)), 0x0040),
                           __byte_perm(__float_as_uint(p2lo(t23)), __float_as_uint(p2hi(t23)), 0x0040),
                           0x5410);
    }
    return make_uint2(w[0], w[1]);
}

template <int N>
__device__ __forceinline__ uint2 codes8_clamp(const uint64_t (&x2)[N], int k0, float rr) {
    uint32_t w[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint64_t* pv = x2 + k0 + 2 * i;
        w[i] = pack_clamp4(__fmul_rn(p2lo(pv[0]), rr), __fmul_rn(p2hi(pv[0]), rr),
                           __fmul_rn(p2lo(pv[1]), rr), __fmul_rn(p2hi(pv[1]), rr));
    }
    return make_uint2(w[0], w[1]);
}

// Eight E2M1 codes (round to nearest even, saturating) of the four value
// pairs, element 2i in the low nibble of byte i.
__device__ __forceinline__ uint32_t e2m1x8(uint64_t a, uint64_t b, uint64_t c, uint64_t d) {
    uint32_t w;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(w)
        : "f"(p2lo(a)), "f"(p2hi(a)), "f"(p2lo(b)), "f"(p2hi(b)), "f"(p2lo(c)), "f"(p2hi(c)),
          "f"(p2lo(d)), "f"(p2hi(d)));
    return w;
}

// ---------------------------------------------------------------- kernel
// Persistent CTAs of 512 threads; CTA c takes tiles c, c + G, c + 2G, ...
// (G = gridDim.x, odd when K and V alternate, so every CTA gets both
// kinds) through a ring of kQStages shared-memory tiles: tile i + kQStages
// is issued as soon as every thread has read tile i. Thread 0 builds the
// descriptor of tile i + kQStages at the top of iteration i, while the
// copies of tile i land. The first K or V tile a CTA issues waits for the
// statistics kernel (griddepcontrol.wait).
// MX = true: Q and K tiles are written as MXFP4 instead of INT8: per row and
// block of 32 consecutive elements (the four threads of the row's quad hold
// 8 elements each), a = max |x_hat|, E = floor(log2 a) - 2 clamped to
// [-127, 125] (-127 for a = 0 or a subnormal a), codes
// e2m1_rn_satfinite(x_hat * 2^-E) (an exact power-of-two scaling), scale
// byte E + 127; an all-zero block gets +0 codes. Codes are packed two per
// byte, element 2i in the low nibble; scale bytes go to the tile's 512-byte
// block in the layout the block-scaled MMA reads (row r, block b at
// 16 (r mod 32) + 4 (r div 32) + b; unused blocks of a D = 64 row are 0).
template <int D, bool MX>
__global__ void __launch_bounds__(kQThreads, kQMinCtas) quant_tiles_kernel(QuantJob j) {
    constexpr int kTileElems = kTile * D;
    constexpr int NM = D / 32;                    // Q/K: 8-value chunks per thread
    constexpr int NP = D / 8;                     // Q/K: value pairs per thread
    constexpr int CPR = D / 8;                    // 16-byte chunks per token row
    constexpr int RP = kQThreads / CPR;           // token rows one pass of copies covers
    constexpr int NPASS = kTile / RP;             // copy passes per tile
    // descriptor ring: the slot written at the top of iteration i last held
    // tile i - 2's descriptor, whose readers all passed iteration i - 1's
    // first barrier
    constexpr int NSLOT = kQStages + 2;
    extern __shared__ __align__(128) unsigned char quant_smem[];
    uint16_t* tiles = reinterpret_cast<uint16_t*>(quant_smem);                                        // [kQStages][kTileElems]
    float* stat = reinterpret_cast<float*>(quant_smem + kQStages * kTileElems * sizeof(uint16_t));  // [kQStages][D]
    __shared__ __align__(16) float wmax[kQThreads / 32];
    __shared__ __align__(16) float zeros[D];
    __shared__ TileDesc tdesc[NSLOT];

    const int n_tiles = j.nq + j.nk + j.nv;
    const int G = gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // this thread's share of every tile copy: chunk cc of rows cr + k RP
    // (RP is even, so those rows share cr's swizzle)
    const int cr = tid / CPR, cc = tid % CPR;
    const int soff = cr * D + 8 * swz(cr, cc);
    bool stats_ready = false;

    // one copy group per tile slot and thread (empty past the end, and the
    // tile part empty for gathered views), so "kQStages - 1 groups pending"
    // always means "the current tile has landed"
    auto start = [&](int t, int slot, int buf) {
        if (t < n_tiles) {
            const TileDesc& d = tdesc[slot];
            if (d.kind != kKindQ) {
                if (!stats_ready) {
                    pdl_wait();                   // the statistics are complete and visible
                    stats_ready = true;
                }
                if (tid < D / 4) cp_async16(stat + buf * D + 4 * tid, d.stat + 4 * tid);
            }
            if (d.vec) {
                const int64_t rs = d.rstride;
                const uint16_t* s0 = d.src + (int64_t)cr * rs + 8 * cc;
                uint16_t* t0 = tiles + buf * kTileElems + soff;
                const int nrows = d.nrows;
#pragma unroll
                for (int k = 0; k < NPASS; ++k)
                    if (cr + k * RP < nrows) cp_async16(t0 + k * RP * D, s0 + (int64_t)(k * RP) * rs);
            }
        }
        cp_async_commit();
    };

    if (tid < D) zeros[tid] = 0.0f;
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < kQStages; ++s)
            if (blockIdx.x + s * G < n_tiles) tdesc[s] = make_desc<D, MX>(blockIdx.x + s * G, j);
    }
    __syncthreads();
#pragma unroll
    for (int s = 0; s < kQStages; ++s) start(blockIdx.x + s * G, s, s);

    for (int it = 0, t = blockIdx.x; t < n_tiles; ++it, t += G) {
        const int buf = it % kQStages;
        const int slot = it % NSLOT;
        const int nslot = (it + kQStages) % NSLOT;
        const int tn = t + kQStages * G;
        if (tid == 0 && tn < n_tiles) tdesc[nslot] = make_desc<D, MX>(tn, j);
        uint16_t* tile = tiles + buf * kTileElems;
        const float* st = stat + buf * D;
        const TileDesc& d = tdesc[slot];
        const int kind = d.kind, nrows = d.nrows;
        if (t + G >= n_tiles) pdl_launch_dependents();   // this CTA's last tile
        cp_async_wait<kQStages - 1>();           // this thread's copies of tile t are in
        if (!d.vec) gather_tile<D>(view_of(j, kind), d.b, d.h, d.l0, nrows, tile);
        __syncthreads();                         // everyone's copies (and descriptors) are in

        if (kind == kKindV) {
            // thread (p, g): channels 2p, 2p + 1 over tokens [g TT, g TT + TT)
            constexpr int P = D / 2, NG = kQThreads / P, TT = kTile / NG;
            const int p = tid % P, g = tid / P;
            const uint64_t r2 = *reinterpret_cast<const uint64_t*>(st + 2 * p);
            // the pair's offset in even and in odd token rows
            const int ce = 8 * (p >> 2) + 2 * (p & 3), co = 8 * ((p >> 2) ^ 4) + 2 * (p & 3);
            const uint16_t* base = tile + g * TT * D;
            const int nvalid = nrows - g * TT;
            uint32_t w0[TT / 4], w1[TT / 4];
#pragma unroll
            for (int t4 = 0; t4 < TT / 4; ++t4) {
                float y0[4], y1[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tok = 4 * t4 + i;
                    uint32_t u = *reinterpret_cast<const uint32_t*>(base + tok * D + ((i & 1) ? co : ce));
                    u = tok < nvalid ? u : 0u;
                    const uint64_t y = p2mul(p2(bf16_bits_to_f32(u & 0xFFFFu), __uint_as_float(u & 0xFFFF0000u)), r2);
                    y0[i] = p2lo(y);
                    y1[i] = p2hi(y);
                }
                w0[t4] = e4m3x2_rn_satfinite(y0[0], y0[1]) | (uint32_t(e4m3x2_rn_satfinite(y0[2], y0[3])) << 16);
                w1[t4] = e4m3x2_rn_satfinite(y1[0], y1[1]) | (uint32_t(e4m3x2_rn_satfinite(y1[2], y1[3])) << 16);
            }
            __syncthreads();                     // every read of the buffer is done
            start(tn, nslot, buf);
            // two contiguous runs of TT bytes in the transposed output
            const int64_t lpad = d.lpad;
            uint8_t* dst = static_cast<uint8_t*>(d.out) + 2 * p * lpad + g * TT;
            if constexpr (TT == 16) {
                *reinterpret_cast<uint4*>(dst) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                *reinterpret_cast<uint4*>(dst + lpad) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
            } else {
                static_assert(TT == 8, "token run of 8 or 16");
                *reinterpret_cast<uint2*>(dst) = make_uint2(w0[0], w0[1]);
                *reinterpret_cast<uint2*>(dst + lpad) = make_uint2(w1[0], w1[1]);
            }
        } else {
            // quad (r, sub): token row r, elements 32 m + 8 sub + i
            const bool isK = kind == kKindK;
            const int r = tid >> 2, sub = tid & 3;
            const bool valid = r < nrows;
            const uint16_t* row = tile + r * D;
            uint64_t x2[NP];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                uint4 u = *reinterpret_cast<const uint4*>(row + 8 * swz(r, 4 * m + sub));
                if (!valid) u = make_uint4(0, 0, 0, 0);      // rows past L are the zero padding
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    x2[4 * m + e] = p2(bf16_bits_to_f32(w[e] & 0xFFFFu), __uint_as_float(w[e] & 0xFFFF0000u));
            }
            if (isK) {
                const float* mean = valid ? st : zeros;       // padding rows stay zero
#pragma unroll
                for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        x2[4 * m + e] = p2sub(x2[4 * m + e],
                                              *reinterpret_cast<const uint64_t*>(mean + 32 * m + 8 * sub + 2 * e));
            }
            quad_butterfly<D>(x2, sub);

            if constexpr (MX) {
                // every read of the buffer is done once all threads are here
                __syncthreads();
                start(tn, nslot, buf);
                uint8_t* codes = static_cast<uint8_t*>(d.out) + r * (D / 2) + 4 * sub;
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    float a = 0.0f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) a = fmax3(a, fabsf(p2lo(x2[4 * m + e])), fabsf(p2hi(x2[4 * m + e])));
                    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
                    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
                    const int ef = static_cast<int>(__float_as_uint(a) >> 23);      // a >= +0
                    const int E = ef == 0 ? -127 : max(ef - 129, -127);
                    const float sc = __uint_as_float(static_cast<uint32_t>(127 - E) << 23);   // 2^-E
                    const uint64_t sc2 = p2(sc, sc);
                    uint32_t w = e2m1x8(p2mul(x2[4 * m], sc2), p2mul(x2[4 * m + 1], sc2),
                                        p2mul(x2[4 * m + 2], sc2), p2mul(x2[4 * m + 3], sc2));
                    if (a == 0.0f) w = 0u;
                    if (valid) *reinterpret_cast<uint32_t*>(codes + 16 * m) = w;
                    else *reinterpret_cast<uint32_t*>(codes + 16 * m) = 0u;
                    if (sub == 0) d.sf[16 * (r & 31) + 4 * (r >> 5) + m] = valid ? static_cast<uint8_t>(E + 127) : 0;
                }
                if (D == 64 && sub == 0) {
                    d.sf[16 * (r & 31) + 4 * (r >> 5) + 2] = 0;
                    d.sf[16 * (r & 31) + 4 * (r >> 5) + 3] = 0;
                }
                continue;
            }

            float a = 0.0f;
#pragma unroll
            for (int k = 0; k < NP; ++k) a = fmax3(a, fabsf(p2lo(x2[k])), fabsf(p2hi(x2[k])));
            // a >= +0, so the bit patterns order like the values
            const unsigned am = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
            if (lane == 0) wmax[warp] = __uint_as_float(am);
            __syncthreads();                     // every row has left the buffer; warp maxima are in
            start(tn, nslot, buf);
            const int blk = d.blk;
            const int wpb = blk >> 3;            // warps per quantisation block (8 rows a warp): 4, 8, 16
            const float4* wm = reinterpret_cast<const float4*>(wmax + (warp & ~(wpb - 1)));
            float amax = 0.0f;
            for (int i = 0; i < wpb / 4; ++i) {
                const float4 v4 = wm[i];
                amax = fmax3(amax, v4.x, v4.y);
                amax = fmax3(amax, v4.z, v4.w);
            }
            float s = 0.0f, rr = 0.0f;
            if (amax != 0.0f) {
                s = __fdiv_rn(amax, 127.0f);
                rr = __fdiv_rn(127.0f, amax);
            }
            if (valid && sub == 0 && (r & (blk - 1)) == 0) d.scale[r / blk] = s;
            int8_t* dst = static_cast<int8_t*>(d.out) + r * D + 8 * sub;
            if (isfinite(rr)) {
#pragma unroll
                for (int m = 0; m < NM; ++m) *reinterpret_cast<uint2*>(dst + 32 * m) = codes8_magic(x2, 4 * m, rr);
            } else {
#pragma unroll
                for (int m = 0; m < NM; ++m) *reinterpret_cast<uint2*>(dst + 32 * m) = codes8_clamp(x2, 4 * m, rr);
            }
        }
    }
}

template <int D>
size_t tiles_smem_bytes() {
    return (size_t)kQStages * ((size_t)kTile * D * sizeof(uint16_t) + D * sizeof(float));
}

// The statistics of the given tensors, then the tiles of the given tensors;
// null views are skipped. ws: [B * Hk][D] fp32 K means (when k), then
// [B * Hk][D] fp32 V multipliers (when v).
// MX = true: Q and K as MXFP4 (q4 / q_sf / k4 / k_sf; no V, no INT8 outputs)
template <int D, bool MX = false>
cudaError_t launch_quant_d(const View4* q, const View4* k, const View4* v, int blk_q, int blk_k,
                           int8_t* q8, float* q_scale, int8_t* k8, float* k_scale, float* k_mean,
                           uint8_t* v8t, float* v_scale, void* ws, cudaStream_t s,
                           uint8_t* q4 = nullptr, uint8_t* q_sf = nullptr, uint8_t* k4 = nullptr,
                           uint8_t* k_sf = nullptr) {
    const View4 none = {};
    const int nkh = k ? (int)(k->size[0] * k->size[1]) : 0;
    const int nvh = v ? (int)(v->size[0] * v->size[1]) : 0;
    float* wsf = static_cast<float*>(ws);

    StatsJob sj;
    sj.k = k ? *k : none;
    sj.v = v ? *v : none;
    sj.nk = nkh;
    sj.nv = nvh;
    sj.kvec = k ? (int)view_vec8(*k) : 0;
    sj.vvec = v ? (int)view_vec8(*v) : 0;
    sj.k_mean_ws = wsf;
    sj.k_mean = k_mean;
    sj.v_rmul_ws = wsf + (size_t)nkh * D;
    sj.v_scale = v_scale;
    if (nkh + nvh > 0) {
        cudaError_t e = cudaFuncSetAttribute(head_stats_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)stat_smem_bytes<D>());
        if (e != cudaSuccess) return e;
        head_stats_kernel<D><<<kStatCluster * (nkh + nvh), kStatThreads, stat_smem_bytes<D>(), s>>>(sj);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }

    QuantJob j;
    j.q = q ? *q : none;
    j.k = sj.k;
    j.v = sj.v;
    j.nq = q ? (int)(q->size[0] * q->size[1] * ceil_div(q->size[2], kTile)) : 0;
    j.nk = k ? (int)(nkh * ceil_div(k->size[2], kTile)) : 0;
    j.nv = v ? (int)(nvh * ceil_div(v->size[2], kTile)) : 0;
    j.blk_q = blk_q;
    j.blk_k = blk_k;
    j.qvec = q ? (int)view_vec8(*q) : 0;
    j.kvec = sj.kvec;
    j.vvec = sj.vvec;
    j.k_mean_ws = sj.k_mean_ws;
    j.v_rmul_ws = sj.v_rmul_ws;
    j.q8 = q8;
    j.q_scale = q_scale;
    j.k8 = k8;
    j.k_scale = k_scale;
    j.v8t = v8t;
    j.q4 = q4;
    j.q_sf = q_sf;
    j.k4 = k4;
    j.k_sf = k_sf;
    const int n_tiles = j.nq + j.nk + j.nv;
    if (n_tiles == 0) return cudaSuccess;

    auto kern = quant_tiles_kernel<D, MX>;
    const size_t smem = tiles_smem_bytes<D>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kQThreads, smem);
    if (e != cudaSuccess) return e;
    int grid = std::min(n_tiles, num_sms() * std::max(1, per_sm));
    if (j.nk > 0 && j.nv > 0 && grid > 1 && (grid & 1) == 0) --grid;   // CTAs alternate K and V tiles
    e = launch_pdl(kern, dim3(grid), dim3(kQThreads), smem, s, j);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename F>
cudaError_t by_head_dim(int D, F&& f) {
    return D == 128 ? f(std::integral_constant<int, 128>()) : f(std::integral_constant<int, 64>());
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

size_t quant_qkv_ws_bytes(int B, int Hk, int Lk, int D) {
    return quant_qk_ws_bytes(B, Hk, Lk, D) + quant_v_ws_bytes(B, Hk, Lk, D);
}

cudaError_t launch_quant_qk(const View4& q, const View4& k, int blk_q, int blk_k, int8_t* q8,
                            float* q_scale, int8_t* k8, float* k_scale, float* k_mean, void* ws,
                            cudaStream_t s, bool with_q) {
    return by_head_dim((int)k.size[3], [&](auto d) {
        return launch_quant_d<decltype(d)::value>(with_q ? &q : nullptr, &k, nullptr, blk_q, blk_k, q8,
                                                  q_scale, k8, k_scale, k_mean, nullptr, nullptr, ws, s);
    });
}

cudaError_t launch_quant_v(const View4& v, uint8_t* v8t, float* v_scale, void* ws,
                           cudaStream_t s) {
    return by_head_dim((int)v.size[3], [&](auto d) {
        return launch_quant_d<decltype(d)::value>(nullptr, nullptr, &v, 0, 0, nullptr, nullptr, nullptr,
                                                  nullptr, nullptr, v8t, v_scale, ws, s);
    });
}

cudaError_t launch_quant_qkv(const View4& q, const View4& k, const View4& v, int blk_q, int blk_k,
                             int8_t* q8, float* q_scale, int8_t* k8, float* k_scale, float* k_mean,
                             uint8_t* v8t, float* v_scale, void* ws, cudaStream_t s) {
    return by_head_dim((int)k.size[3], [&](auto d) {
        return launch_quant_d<decltype(d)::value>(&q, &k, &v, blk_q, blk_k, q8, q_scale, k8, k_scale,
                                                  k_mean, v8t, v_scale, ws, s);
    });
}

cudaError_t launch_quant_qk_mx(const View4& q, const View4& k, uint8_t* q4, uint8_t* q_sf, uint8_t* k4,
                               uint8_t* k_sf, float* k_mean, void* ws, cudaStream_t s) {
    return by_head_dim((int)k.size[3], [&](auto d) {
        return launch_quant_d<decltype(d)::value, true>(&q, &k, nullptr, 32, 32, nullptr, nullptr, nullptr,
                                                        nullptr, k_mean, nullptr, nullptr, ws, s, q4, q_sf,
                                                        k4, k_sf);
    });
}

}  // namespace sage
// ---------------------------------------------------------------- no-allocation variant
// sage_quant_qk_noalloc: the same Q/K smoothing + rotation + INT8 quantisation
// as sage_quant_qk, for callers that cannot allocate device memory at the
// point of the call -- for instance a serving loop whose device memory is
// budgeted once at start-up, or code that must not risk the implicit device
// synchronisation that cudaMalloc / cudaFree can cause. Its scratch -- the
// fp32 K mean of every (b, kv head), B * Hk * D * 4 bytes, written by the
// statistics kernel and read by the tile kernel -- lives in the fixed array
// below instead of a caller workspace.
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
