// attn_mx.cu -- quantised attention forward with MXFP4 Q and K for sm_100a
// (the fav3_sage_mxfp4 variant of "Sage v2 improvements": Q and K rotated by
// the Hadamard matrix, then E2M1 codes with one e8m0 scale per 32 elements
// of a row; "[FlyDSL] [Misc] pa_decode ...": P keeps the E4M3 format).
//
// S = Q4 K4^T is one block-scaled tcgen05 MMA per 64 head-dim elements
// (kind::mxf4, scales of 32-element blocks read from TMEM, fp32 into TMEM),
// so the logit is S * softmax_scale / D with no per-row or per-key scale
// left to apply. The rest of the per-tile sequence is that of
// attn_fwd_kernel: running max, alpha rescale of O, accumulate_d on the
// unquantised exponentials, P8 = e4m3(448 * 2^(y - m)), PV in FP8 with V per
// channel, out = bf16(O * v_scale / (448 d)).
//
// One CTA owns one 128-row query tile of one (b, h). TMEM (512 columns):
// S double-buffered at [0, 128) and [128, 256), O at [256, 256 + D), the
// query tile's scale factors at [448, 452), the current key tile's at
// [452, 456). Roles (288 threads):
//   warps 0-7  softmax: warp w serves key columns 64 (w >> 2) .. + 64 of each
//              128-key tile and TMEM lanes 32 (w & 3) .. + 32; the two warps of
//              a row exchange half-row maxima (and, at the end, half-row sums)
//              through shared memory on a two-arrival mbarrier. S is read from
//              TMEM twice per tile (a max pass, then the exponentials), 32
//              columns at a time, and its buffer is released after the second
//              pass: QK of the next tile runs into the other buffer meanwhile.
//   warp 8     control, one thread: TMA loads (Q4 tile and its scales once;
//              a ring of K4 tiles with their scales and V^T tiles), the
//              tcgen05.cp copies of the scales into TMEM and every MMA, in
//              one in-order loop. tcgen05 operations of one thread run in
//              issue order, so each key tile's scales can be copied into the
//              same TMEM columns just before its QK.
// Every mbarrier wait is bounded; on timeout the CTA records an error word,
// raises a CTA-wide abort flag, drains its own MMAs and returns.
#include <climits>
#include <cstring>

#include <cuda.h>
#include <cuda_bf16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {

unsigned read_clear_attn_mx_error();

namespace {

__device__ unsigned g_attn_mx_err;

constexpr int BM = 128;            // query rows per CTA
constexpr int BN = 128;            // keys per tile
constexpr int BH = BN / 2;         // key columns per softmax warp
constexpr int kSoftWarps = 8;
constexpr int kCtrlWarp = 8;
constexpr int kThreads = 32 * (kSoftWarps + 1);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;   // log2(FP8_MAX of e4m3)
constexpr uint32_t kSfaCol = 448, kSfbCol = 452;
constexpr int kPolyEvery = 8;      // as in attn_fwd.cu: every 8th key pair on the FMA pipe

template <int D>
struct Cfg {
    static constexpr int kStages = 4;
    static constexpr int kRowBytes = D / 2;                 // packed E2M1 row
    static constexpr int kQBytes = BM * kRowBytes;
    static constexpr int kKBytes = BN * kRowBytes;
    static constexpr int kSfBytes = 512;                    // scales of 128 rows
    static constexpr int kVBytes = D * BN;
    static constexpr int kPBytes = BM * BN;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = 8192;                      // Q tile (<= 8 KB) rounded to 8 KB
    static constexpr int kOffV = kOffK + kStages * kKBytes;
    static constexpr int kOffP = kOffV + kStages * kVBytes; // [2] tiles
    static constexpr int kOffSfq = kOffP + 2 * kPBytes;
    static constexpr int kOffSfk = kOffSfq + kSfBytes;      // [kStages]
    static constexpr int kOffBar = kOffSfk + kStages * kSfBytes;
    static constexpr int kBarQ = 0;
    static constexpr int kBarKFull = 1;
    static constexpr int kBarKEmpty = kBarKFull + kStages;
    static constexpr int kBarVFull = kBarKEmpty + kStages;
    static constexpr int kBarVEmpty = kBarVFull + kStages;
    static constexpr int kBarSFull = kBarVEmpty + kStages;  // [2 buffers]
    static constexpr int kBarSEmpty = kBarSFull + 2;        // [2 buffers], 8 warp arrivals
    static constexpr int kBarPFull = kBarSEmpty + 2;        // 8 warp arrivals
    static constexpr int kBarODone = kBarPFull + 1;
    static constexpr int kBarX = kBarODone + 1;             // [4 row quarters], 2 warp arrivals
    static constexpr int kBarFinal = kBarX + 4;
    static constexpr int kNumBars = kBarFinal + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kOffVs = kOffMisc + 16;
    static constexpr int kOffX = kOffVs + D * 4;            // [2 parity][2 half][128] fp32
    static constexpr int kSmemBytes = kOffX + 2 * 2 * BM * 4 + 1024;
    static_assert(kQBytes <= 8192, "query tile");
    static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0, "alignment");
    static_assert(kOffSfq % 16 == 0 && kOffSfk % 16 == 0, "bulk copy alignment");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct Params {
    const uint8_t* q_sf;
    const uint8_t* k_sf;
    const float* v_scale;
    __nv_bfloat16* out;
    int64_t os0, os1, os2, os3;
    int H, Hk, Lq, Lk, LpadQ, LpadK;
    float logit_scale_log2;        // softmax_scale / D * log2(e)
    int heavy_first;
    int out_vec;
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// Shared-memory descriptor of a K-major operand tile with rows of
// `row_bytes` (128, 64 or 32) stored with the matching TMA swizzle: 8-row
// core groups 8 * row_bytes apart (SBO), version 1, base offset 0.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr, int row_bytes) {
    const uint64_t mode = row_bytes == 128 ? 2 : (row_bytes == 64 ? 4 : 6);
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>((8u * row_bytes) >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= mode << 61;
    return d;
}

// Descriptor of a 512-byte scale-factor block as the tcgen05.cp source: 32
// rows of 16 bytes, no swizzle, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(128 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    return d;
}

// Copy a scale-factor block from shared memory to TMEM columns [taddr,
// taddr + 4): row i of the block (16 bytes) to lane i of every lane quarter.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

// Instruction descriptor of the block-scaled E2M1 MMA (kind::mxf4, e8m0
// scales, 32-element blocks, K = 64): A and B K-major, M = 128, N = 128;
// sf_id picks the scale bytes (sf_id, sf_id + 1) of each row's 4-byte word.
__host__ __device__ constexpr uint32_t idesc_mxf4(uint32_t sf_id) {
    return (sf_id << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
           (1u << 23) | (static_cast<uint32_t>(BM >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}

// Four e4m3 codes (RN, satfinite) of e0..e3 in one word, e0 in byte 0.
__device__ __forceinline__ uint32_t e4m3x4(float e0, float e1, float e2, float e3) {
    uint32_t w;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(w)
        : "f"(e0), "f"(e1), "f"(e2), "f"(e3));
    return w;
}

// Max of 32 consecutive scores; MASK: keys j0 + k > jlim count as -inf.
template <bool MASK>
__device__ __forceinline__ float chunk_max(const uint32_t (&s)[32], int j0, int jlim) {
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        float x0 = __uint_as_float(s[2 * k]), x1 = __uint_as_float(s[2 * k + 1]);
        if (MASK) {
            x0 = (j0 + 2 * k <= jlim) ? x0 : -INFINITY;
            x1 = (j0 + 2 * k + 1 <= jlim) ? x1 : -INFINITY;
        }
        mx[k & 3] = fmax3(mx[k & 3], x0, x1);
    }
    return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// accumulate_d and RS_32_to_8 for 32 keys of a row: base-2 logits
// S * c + cofs in place (one f32x2 FMA per key pair), exponentials, the sum,
// e4m3 packing and the P8 stores of 16-byte chunks c0, c0 + 1 of the row
// (128B-swizzled K-major: chunk c of row r at c ^ (r & 7)).
template <bool MASK>
__device__ __forceinline__ float chunk_exp(uint32_t (&s)[32], float c, float cofs, int j0, int jlim,
                                           uint8_t* prow, int r, int c0) {
    const uint64_t c2 = f2_pack(c, c), cofs2 = f2_pack(cofs, cofs);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        float a0, a1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), c2, cofs2), a0, a1);
        if (MASK) {
            a0 = (j0 + 2 * k <= jlim) ? a0 : -INFINITY;
            a1 = (j0 + 2 * k + 1 <= jlim) ? a1 : -INFINITY;
        }
        s[2 * k] = __float_as_uint(a0);
        s[2 * k + 1] = __float_as_uint(a1);
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        float e0, e1;
        if (kPolyEvery > 0 && k % kPolyEvery == kPolyEvery - 1) {
            exp2_poly_x2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1]), e0, e1);
        } else {
            e0 = ex2_approx(__uint_as_float(s[2 * k]));
            e1 = ex2_approx(__uint_as_float(s[2 * k + 1]));
        }
        s[2 * k] = __float_as_uint(e0);
        s[2 * k + 1] = __float_as_uint(e1);
    }
    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        uint32_t pk[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t* e = s + 16 * cc + 4 * q;
            acc[q] = f2_add(acc[q], f2_pack(__uint_as_float(e[0]), __uint_as_float(e[1])));
            acc[q] = f2_add(acc[q], f2_pack(__uint_as_float(e[2]), __uint_as_float(e[3])));
            pk[q] = e4m3x4(__uint_as_float(e[0]), __uint_as_float(e[1]), __uint_as_float(e[2]),
                           __uint_as_float(e[3]));
        }
        *reinterpret_cast<uint4*>(prow + (((c0 + cc) ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    const uint64_t t2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
    float r0, r1;
    f2_unpack(t2, r0, r1);
    return r0 + r1;
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_mx_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
    using C = Cfg<D>;
    constexpr int DH = D / 2;                       // output columns per softmax warp
    constexpr int KK = D / 64;                      // block-scaled MMAs per QK (K = 64 each)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    int bh, qt;
    if (p.heavy_first) {
        bh = blockIdx.x;
        qt = gridDim.y - 1 - blockIdx.y;
    } else {
        qt = blockIdx.x;
        bh = blockIdx.y;
    }
    const int b = bh / p.H, h = bh % p.H;
    const int bhk = b * p.Hk + h / (p.H / p.Hk);
    const int q_row0 = qt * BM;
    int kv_end = p.Lk;
    if (CAUSAL) kv_end = max(0, min(kv_end, q_row0 + BM + (p.Lk - p.Lq)));
    const int n_t = (kv_end + BN - 1) / BN;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i == C::kBarSEmpty || i == C::kBarSEmpty + 1 || i == C::kBarPFull) cnt = kSoftWarps;
            if (i >= C::kBarX && i < C::kBarX + 4) cnt = 2;
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kCtrlWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    float* vs_s = reinterpret_cast<float*>(smem + C::kOffVs);
    float* xch = reinterpret_cast<float*>(smem + C::kOffX);       // [parity][half][128]
    pdl_wait();
    for (int i = threadIdx.x; i < D; i += kThreads) vs_s[i] = __ldg(&p.v_scale[(int64_t)bhk * D + i]);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kCtrlWarp) {
        // ---------------------------------------------------------- control
        if (lane == 0 && n_t > 0) {
            const uint32_t sQ = smem_u32(smem + C::kOffQ);
            const uint32_t sK = smem_u32(smem + C::kOffK);
            const uint32_t sV = smem_u32(smem + C::kOffV);
            const uint32_t sP = smem_u32(smem + C::kOffP);
            constexpr uint32_t kIdescPV = umma_idesc(1, 0, BM, D);    // e4m3 x e4m3 -> f32
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&bars[C::kBarQ], C::kQBytes + C::kSfBytes);
            tma_load_2d(smem + C::kOffQ, &tmQ, &bars[C::kBarQ], 0, bh * p.LpadQ + q_row0);
            bulk_load(smem + C::kOffSfq, p.q_sf + ((int64_t)bh * p.LpadQ + q_row0) / BM * C::kSfBytes,
                      C::kSfBytes, &bars[C::kBarQ]);
            auto load = [&](int t) -> bool {
                const int s = t % C::kStages;
                const uint32_t ph = (t / C::kStages) & 1;
                if (!mbar_wait(&bars[C::kBarKEmpty + s], ph ^ 1, abort_flag, &g_attn_mx_err, 1)) return false;
                mbar_arrive_expect_tx(&bars[C::kBarKFull + s], C::kKBytes + C::kSfBytes);
                tma_load_2d(smem + C::kOffK + s * C::kKBytes, &tmK, &bars[C::kBarKFull + s], 0,
                            bhk * p.LpadK + t * BN);
                bulk_load(smem + C::kOffSfk + s * C::kSfBytes,
                          p.k_sf + ((int64_t)bhk * p.LpadK + t * BN) / BN * C::kSfBytes, C::kSfBytes,
                          &bars[C::kBarKFull + s]);
                if (!mbar_wait(&bars[C::kBarVEmpty + s], ph ^ 1, abort_flag, &g_attn_mx_err, 2)) return false;
                mbar_arrive_expect_tx(&bars[C::kBarVFull + s], C::kVBytes);
                tma_load_2d(smem + C::kOffV + s * C::kVBytes, &tmV, &bars[C::kBarVFull + s], t * BN, bhk * D);
                return true;
            };
            // S(t) = Q4 K4(t)^T into S buffer t & 1, once the softmax has
            // released that buffer (tile t - 2); the key tile's scales are
            // copied into TMEM just before (same thread: in order)
            auto issue_qk = [&](int t) -> bool {
                const int s = t % C::kStages;
                const uint32_t ph = (t / C::kStages) & 1;
                if (!mbar_wait(&bars[C::kBarKFull + s], ph, abort_flag, &g_attn_mx_err, 6)) return false;
                if (!mbar_wait(&bars[C::kBarSEmpty + (t & 1)], (t >> 1) & 1, abort_flag, &g_attn_mx_err, 7))
                    return false;
                tc_fence_after();
                tmem_cp_sf(tmem + kSfbCol, desc_sf(smem_u32(smem + C::kOffSfk + s * C::kSfBytes)));
                const uint64_t qdesc = desc_kmajor(sQ, C::kRowBytes);
                const uint64_t kdesc = desc_kmajor(sK + s * C::kKBytes, C::kRowBytes);
#pragma unroll
                for (int kk = 0; kk < KK; ++kk)
                    mma_mxf4(tmem + 128 * (t & 1), qdesc + 2 * kk, kdesc + 2 * kk, idesc_mxf4(2 * kk),
                             tmem + kSfaCol, tmem + kSfbCol, kk > 0 ? 1u : 0u);
                mma_commit(&bars[C::kBarSFull + (t & 1)]);
                mma_commit(&bars[C::kBarKEmpty + s]);
                return true;
            };
            auto issue_pv = [&](int t) -> bool {
                const int s = t % C::kStages;
                const uint32_t ph = (t / C::kStages) & 1;
                if (!mbar_wait(&bars[C::kBarVFull + s], ph, abort_flag, &g_attn_mx_err, 3)) return false;
                if (!mbar_wait(&bars[C::kBarPFull], t & 1, abort_flag, &g_attn_mx_err, 4)) return false;
                tc_fence_after();
                const uint64_t vdesc = umma_desc_kmajor(sV + s * C::kVBytes, 128);
                const uint64_t pdesc = umma_desc_kmajor(sP + (t & 1) * C::kPBytes, 128);
#pragma unroll
                for (int kk = 0; kk < BN / 32; ++kk)
                    mma_f8_ss(tmem + 256, pdesc + 2 * kk, vdesc + 2 * kk, kIdescPV, (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bars[C::kBarODone]);
                mma_commit(&bars[C::kBarVEmpty + s]);
                return true;
            };
            bool ok = true;
            for (int t = 0; ok && t < min(n_t, C::kStages); ++t) ok = load(t);
            if (ok) ok = mbar_wait(&bars[C::kBarQ], 0, abort_flag, &g_attn_mx_err, 5);
            if (ok) {
                tc_fence_after();
                tmem_cp_sf(tmem + kSfaCol, desc_sf(smem_u32(smem + C::kOffSfq)));
                ok = issue_qk(0);
            }
            for (int t = 0; ok && t < n_t; ++t) {
                if (t + 1 < n_t) ok = issue_qk(t + 1);
                if (ok) ok = issue_pv(t);
                if (ok && t + C::kStages < n_t) ok = load(t + C::kStages);
            }
            mma_commit(&bars[C::kBarFinal]);
            mbar_wait(&bars[C::kBarFinal], 0, abort_flag, &g_attn_mx_err, 8);
        }
    } else {
        // ---------------------------------------------------------- softmax
        const int hf = warp >> 2, ww = warp & 3;
        const int r = ww * 32 + lane;
        const int i = q_row0 + r;
        const bool valid = i < p.Lq;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(ww * 32) << 16);
        const uint32_t o_col = 256 + hf * DH;
        const float c = p.logit_scale_log2;
        int jlim = p.Lk - 1;
        if (CAUSAL && valid) jlim = min(jlim, i + (p.Lk - p.Lq));
        uint64_t* xbar = &bars[C::kBarX + ww];

        // both S buffers start out free
        if (n_t > 0) {
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[C::kBarSEmpty]);
                mbar_arrive(&bars[C::kBarSEmpty + 1]);
            }
        }
        float m = -INFINITY, dsum = 0.0f;
        bool ok = true;
        for (int t = 0; t < n_t; ++t) {
            const int bf = t & 1;
            ok = warp_all(mbar_wait(&bars[C::kBarSFull + bf], (t >> 1) & 1, abort_flag, &g_attn_mx_err, 9));
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_col = 128 * bf + hf * BH;
            const int j0 = t * BN + hf * BH;
            const bool need_mask = __any_sync(0xffffffffu, j0 + BH - 1 > jlim);
            // pass 1: the half row's maximum of S (c > 0 keeps the order)
            float mt = -INFINITY;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t sv[32];
                tmem_ld32(lane_addr + s_col + 32 * cc, sv);
                tmem_wait_ld(sv);
                mt = fmaxf(mt, need_mask ? chunk_max<true>(sv, j0 + 32 * cc, jlim)
                                         : chunk_max<false>(sv, j0 + 32 * cc, jlim));
            }
            mt = mt == -INFINITY ? -INFINITY : mt * c;
            float* xs = xch + (t & 1) * 2 * BM;
            xs[hf * BM + r] = mt;
            __syncwarp();
            if (lane == 0) mbar_arrive(xbar);
            ok = warp_all(mbar_wait(xbar, t & 1, abort_flag, &g_attn_mx_err, 14));
            if (!ok) break;
            mt = fmaxf(mt, xs[(hf ^ 1) * BM + r]);
            const float m_new = fmaxf(m, mt);
            const float msub = (m_new == -INFINITY) ? 0.0f : m_new;
            const float alpha = ex2_approx(m - msub);
            // pass 2: logits, exponentials, sums and P8; then S buffer bf
            // goes back to the control thread
            uint8_t* prow = smem + C::kOffP + (t & 1) * C::kPBytes + r * 128;
            float tsum = 0.0f;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t sv[32];
                tmem_ld32(lane_addr + s_col + 32 * cc, sv);
                tmem_wait_ld(sv);
                tsum += need_mask
                    ? chunk_exp<true>(sv, c, kLog2_448 - msub, j0 + 32 * cc, jlim, prow, r, hf * 4 + 2 * cc)
                    : chunk_exp<false>(sv, c, kLog2_448 - msub, j0 + 32 * cc, jlim, prow, r, hf * 4 + 2 * cc);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[C::kBarSEmpty + bf]);
            dsum = dsum * alpha + tsum;
            if (t > 0) {
                // PV(t - 1) has landed in O; then O *= alpha for this warp's
                // half of the columns (P buffer t & 1 was last read by
                // PV(t - 2), awaited in the previous tile)
                ok = warp_all(mbar_wait(&bars[C::kBarODone], (t - 1) & 1, abort_flag, &g_attn_mx_err, 10));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.0f)) {
                    const uint64_t al2 = f2_pack(alpha, alpha);
#pragma unroll
                    for (int c2 = 0; c2 < DH / 32; ++c2) {
                        uint32_t o[32];
                        tmem_ld32(lane_addr + o_col + 32 * c2, o);
                        tmem_wait_ld(o);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float a0, a1;
                            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2), a0, a1);
                            o[e] = __float_as_uint(a0);
                            o[e + 1] = __float_as_uint(a1);
                        }
                        tmem_st32(lane_addr + o_col + 32 * c2, o);
                    }
                    tmem_wait_st();
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[C::kBarPFull]);
            m = m_new;
        }

        // epilogue: d = the two half rows' sums, out = O * v_scale / (448 d)
        __nv_bfloat16* orow = p.out + b * p.os0 + h * p.os1 + (int64_t)i * p.os2;
        if (ok && n_t > 0) {
            float* xs = xch + (n_t & 1) * 2 * BM;
            xs[hf * BM + r] = dsum;
            __syncwarp();
            if (lane == 0) mbar_arrive(xbar);
            ok = warp_all(mbar_wait(xbar, n_t & 1, abort_flag, &g_attn_mx_err, 15));
            if (ok) dsum += xs[(hf ^ 1) * BM + r];
            if (ok) ok = warp_all(mbar_wait(&bars[C::kBarODone], (n_t - 1) & 1, abort_flag, &g_attn_mx_err, 11));
            if (ok) {
                tc_fence_after();
                const float inv = dsum > 0.0f ? 1.0f / dsum : 0.0f;
#pragma unroll 1
                for (int c2 = 0; c2 < DH / 32; ++c2) {
                    uint32_t o[32];
                    tmem_ld32(lane_addr + o_col + 32 * c2, o);
                    tmem_wait_ld(o);
                    if (valid) {
                        const int d0 = hf * DH + 32 * c2;
                        uint32_t packed[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 vs2 = *reinterpret_cast<const float2*>(vs_s + d0 + e);
                            const __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(o[e]) * (vs2.x * inv),
                                                                            __uint_as_float(o[e + 1]) * (vs2.y * inv));
                            packed[e / 2] = *reinterpret_cast<const uint32_t*>(&pr);
                        }
                        if (p.out_vec) {
                            uint4* dst = reinterpret_cast<uint4*>(orow + d0);
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                dst[q4] = make_uint4(packed[4 * q4], packed[4 * q4 + 1], packed[4 * q4 + 2],
                                                     packed[4 * q4 + 3]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const uint16_t bits16 = (e & 1) ? (packed[e / 2] >> 16) : (packed[e / 2] & 0xFFFFu);
                                *reinterpret_cast<uint16_t*>(orow + (int64_t)(d0 + e) * p.os3) = bits16;
                            }
                        }
                    }
                }
            }
        } else if (n_t == 0 && valid) {
            for (int d = hf * DH; d < hf * DH + DH; ++d) orow[(int64_t)d * p.os3] = __float2bfloat16_rn(0.0f);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kCtrlWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D uint8 tensor map: `rows` rows of `cols` bytes, box {box_cols, box_rows},
// swizzle matching the box's row length (128, 64 or 32 bytes).
bool encode_u8(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_cols,
               uint32_t box_rows) {
    auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = box_cols == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                   : CU_TENSOR_MAP_SWIZZLE_32B;
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool CAUSAL>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const Params& p,
                     dim3 grid, cudaStream_t s) {
    auto kern = attn_mx_kernel<D, CAUSAL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, grid, dim3(kThreads), Cfg<D>::kSmemBytes, s, tq, tk, tv, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_mx(const AttnMxArgs& a, cudaStream_t s) {
    const int LpadQ = static_cast<int>(round_up(a.Lq, kTile));
    const int LpadK = static_cast<int>(round_up(a.Lk, kTile));
    CUtensorMap tq, tk, tv;
    if (!encode_u8(&tq, a.q4, a.D / 2, (uint64_t)a.B * a.H * LpadQ, a.D / 2, BM) ||
        !encode_u8(&tk, a.k4, a.D / 2, (uint64_t)a.B * a.Hk * LpadK, a.D / 2, BN) ||
        !encode_u8(&tv, a.v8t, LpadK, (uint64_t)a.B * a.Hk * a.D, BN, a.D))
        return cudaErrorInvalidValue;
    Params p;
    p.q_sf = a.q_sf;
    p.k_sf = a.k_sf;
    p.v_scale = a.v_scale;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.os0 = a.out_stride[0];
    p.os1 = a.out_stride[1];
    p.os2 = a.out_stride[2];
    p.os3 = a.out_stride[3];
    p.H = a.H;
    p.Hk = a.Hk;
    p.Lq = a.Lq;
    p.Lk = a.Lk;
    p.LpadQ = LpadQ;
    p.LpadK = LpadK;
    p.logit_scale_log2 = a.softmax_scale / static_cast<float>(a.D) * kLog2e;
    p.heavy_first = a.causal ? 1 : 0;
    p.out_vec = (a.out_stride[3] == 1 && a.out_stride[0] % 8 == 0 && a.out_stride[1] % 8 == 0 &&
                 a.out_stride[2] % 8 == 0 && reinterpret_cast<uintptr_t>(a.out) % 16 == 0)
                    ? 1
                    : 0;
    const int nqt = static_cast<int>(ceil_div(a.Lq, BM));
    const dim3 grid = a.causal ? dim3(a.B * a.H, nqt) : dim3(nqt, a.B * a.H);
    if (a.D == 128)
        return a.causal ? launch_t<128, true>(tq, tk, tv, p, grid, s) : launch_t<128, false>(tq, tk, tv, p, grid, s);
    return a.causal ? launch_t<64, true>(tq, tk, tv, p, grid, s) : launch_t<64, false>(tq, tk, tv, p, grid, s);
}

unsigned read_clear_attn_mx_error() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_mx_err, sizeof v) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_attn_mx_err, &zero, sizeof zero);
    return v;
}

}  // namespace sage
