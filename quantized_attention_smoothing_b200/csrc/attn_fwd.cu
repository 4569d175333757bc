// attn_fwd.cu -- quantised attention forward for sm_100a.
//
// One CTA owns two 128-row query tiles of one (b, h) and streams the key
// axis in 128-key tiles. Roles (384 threads):
//   warps 0-3   softmax for query tile 0 (thread = query row = TMEM lane)
//   warps 4-7   softmax for query tile 1
//   warp 8      TMA producer: both Q tiles once, then a ring of K / V^T stages
//   warp 9      MMA issuer (one thread): tcgen05 kind::i8 S = Q8 K8^T into
//               TMEM (int32), tcgen05 kind::f8f6f4 O += P8 V8 into TMEM (fp32)
//   warps 10-11 idle (they complete the register warpgroup of warps 8-9)
// TMEM (512 columns): S_w at [128 w, 128 w + 128), O_w at [256 + 128 w, +D).
// Registers: the CTA launches at 168 per thread; the producer warpgroup
// (warps 8-11) drops to 40 and the softmax warpgroups rise to 232, so a
// thread can hold its whole 128-key score row.
//
// A softmax thread reads its whole score row (128 keys) from TMEM into
// registers and hands the S columns straight back, so the tensor pipe
// computes the next tile's scores while the current ones are converted.
// P8 goes to shared memory (double buffered per query tile), which lets
// PV(t) run while tile t + 1 is converted. MMA issue order per tile t:
//   QK_0(t+1), QK_1(t+1), PV_0(t), PV_1(t)
// so each query tile depends only on its own softmax warps. The two tiles'
// exponential phases take turns (a token passed between the softmax
// warpgroups through bounded mbarriers), so one tile's TMEM traffic, max and
// rescale overlap the other's MUFU work on the SM sub-partitions (the overlap
// "Sage2 SM89 Temporal Pair Experiment" (Candidate) obtains with warp pairs
// on sm_89).
//
// Per 128-key tile the softmax warps follow the page's sequence
//   QK -> update_mdo -> accumulate_d -> RS_32_to_8 -> PV
// with m, d per row in registers, y = acc * (q_scale * k_scale *
// softmax_scale / D * log2 e) (base-2 logits), m' = max(m, max y),
// alpha = 2^(m - m'), d = alpha d + sum 2^(y - m') (before the FP8 cast),
// P8 = e4m3(448 * 2^(y - m')) written to shared memory in the UMMA 128B-swizzled
// K-major layout, and O *= alpha in TMEM whenever alpha != 1 for some row of
// the warp. The epilogue writes bf16(O * v_scale / (448 d)) through the
// caller's strides ("[FlyDSL] [Misc] pa_decode: ...", Changes: P scaled by
// FP8_MAX before the cast, epilogue x 1/FP8_MAX; "sage_attn3" API page: the
// output is written straight into a [B, L, H, D] layout without a copy).
//
// Every mbarrier wait is bounded (see mbar_wait): on timeout the CTA records
// an error word, raises a CTA-wide abort flag, drains its own MMAs and
// returns.
#include <climits>
#include <cstring>

#include <cuda.h>
#include <cuda_bf16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"
#include "quant_rows.cuh"

namespace sage {
namespace {

__device__ unsigned g_attn_err;

constexpr int BM = 128;          // query rows per tile (= TMEM lanes)
constexpr int BN = 128;          // keys per tile
constexpr int QT = 2;            // query tiles per CTA
constexpr int kSoftWarps = 8;    // 2 query tiles x 4 lane quarters
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 32 * (kSoftWarps + 4);
// per-thread registers after the split; 128 * (2 * kSoftRegs + kProdRegs) must
// not exceed kThreads * (registers at launch, 168) or the increase never
// completes
constexpr int kSoftRegs = 232;
constexpr int kProdRegs = 40;
static_assert(128 * (2 * kSoftRegs + kProdRegs) <= kThreads * 168, "register split");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;   // log2(FP8_MAX of e4m3)
constexpr int kMagicI = 0x4B400000;               // bit pattern of 1.5 * 2^23
constexpr float kMagicF = 12582912.0f;            // 1.5 * 2^23
// every kPolyEvery-th key pair takes its exponential from exp2_poly_x2 (FMA
// pipe) instead of the MUFU unit, which relieves the MUFU queue of the warp
// converting its row (0 = never)
constexpr int kPolyEvery = 8;


// K block scales of one head staged in shared memory (larger heads read the
// rest from global memory)
constexpr int kKsSmem = 1024;

template <int D>
struct Cfg {
    static constexpr int kStages = D == 128 ? 3 : 6;
    static constexpr int kQBytes = BM * D;
    static constexpr int kKBytes = BN * D;
    static constexpr int kVBytes = D * BN;
    static constexpr int kPBytes = BM * BN;
    static constexpr int kPBufs = 2;                         // P double buffer per query tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + QT * kQBytes;
    static constexpr int kOffV = kOffK + kStages * kKBytes;
    static constexpr int kOffP = kOffV + kStages * kVBytes;  // [QT][kPBufs] tiles
    static constexpr int kOffBar = kOffP + QT * kPBufs * kPBytes;
    static constexpr int kBarQ = 0;
    static constexpr int kBarKFull = 1;
    static constexpr int kBarKEmpty = kBarKFull + kStages;
    static constexpr int kBarVFull = kBarKEmpty + kStages;
    static constexpr int kBarVEmpty = kBarVFull + kStages;
    static constexpr int kBarSFull = kBarVEmpty + kStages;   // [QT]
    static constexpr int kBarSEmpty = kBarSFull + QT;        // [QT], 4 warp arrivals
    static constexpr int kBarPFull = kBarSEmpty + QT;        // [QT], 4 warp arrivals
    static constexpr int kBarODone = kBarPFull + QT;         // [QT]
    static constexpr int kBarTok = kBarODone + QT;           // [QT], 4 warp arrivals
    static constexpr int kBarFinal = kBarTok + QT;
    static constexpr int kNumBars = kBarFinal + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kOffKs = kOffMisc + 16;             // K block scales of the head
    static constexpr int kOffVs = kOffKs + kKsSmem * 4;      // V channel scales of the head
    static constexpr int kOffQmax = kOffVs + D * 4;          // [8] row-block maxima (in-CTA Q)
    static constexpr int kSmemBytes = kOffQmax + 8 * 4 + 1024; // + runtime alignment
    static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0, "alignment");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct Params {
    const float* q_scale;
    const float* k_scale;
    const float* v_scale;
    __nv_bfloat16* out;
    int64_t os0, os1, os2, os3;
    int H, Hk, Lq, Lk, LpadQ, LpadK, blk_q, blk_k, nbq, nbk;
    int lg_blk_q, lg_blk_k;        // log2 of the (power-of-two) block sizes
    float logit_scale_log2;        // softmax_scale / D * log2(e)
    int heavy_first;
    int out_vec;
};

// The in-CTA Q path: Q rows read as bf16 [B, H, Lq, D] and rotated and
// quantised by the softmax threads (q8 / q_scale unused). A separate,
// trailing kernel parameter, so the separate-Q kernel's code is unchanged.
struct QParams {
    const uint16_t* qbf;
    int64_t qs0, qs1, qs2, qs3;
    int q_vec;                     // 16-byte row loads possible
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// View 32 consecutive registers of a larger per-thread array as one
// tcgen05.ld / st operand.
__device__ __forceinline__ uint32_t (&slice32(uint32_t* base))[32] {
    return *reinterpret_cast<uint32_t(*)[32]>(base);
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

// Max of n consecutive biased scores s[0..n) (fp32 values 1.5 * 2^23 + acc).
// MASK: keys j0 + k > jlim count as -inf.
template <int N, bool MASK>
__device__ __forceinline__ float block_max(const uint32_t* s, int j0, int jlim) {
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
        float x0 = __uint_as_float(s[2 * k]);
        float x1 = __uint_as_float(s[2 * k + 1]);
        if (MASK) {
            x0 = (j0 + 2 * k <= jlim) ? x0 : -INFINITY;
            x1 = (j0 + 2 * k + 1 <= jlim) ? x1 : -INFINITY;
        }
        mx[k & 3] = fmax3(mx[k & 3], x0, x1);
    }
    return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// accumulate_d and RS_32_to_8 for a whole 128-key score row, in three
// sweeps of independent instructions (so a single warp keeps the MUFU unit
// fed): logits in place, exponentials in place, then row sum, e4m3 packing
// and the P8 row store (128B-swizzled K-major: 16-byte chunk c of row r at
// c ^ (r & 7)). Returns the sum of the unquantised exponentials.
template <int NKB, bool MASK>
__device__ __forceinline__ float row_exp(uint32_t (&s)[BN], const float (&kc)[NKB], float cofs,
                                         int j0, int jlim, uint8_t* prow, int r) {
    constexpr int kKeysPerBlk = BN / NKB;
    const uint64_t nmag2 = f2_pack(-kMagicF, -kMagicF);
    const uint64_t cofs2 = f2_pack(cofs, cofs);
#pragma unroll
    for (int k = 0; k < BN / 2; ++k) {
        const float kcc = kc[(2 * k) / kKeysPerBlk];
        const uint64_t x2 = f2_add(f2_pack(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), nmag2);
        float a0, a1;
        f2_unpack(f2_fma(x2, f2_pack(kcc, kcc), cofs2), a0, a1);
        if (MASK) {
            a0 = (j0 + 2 * k <= jlim) ? a0 : -INFINITY;
            a1 = (j0 + 2 * k + 1 <= jlim) ? a1 : -INFINITY;
        }
        s[2 * k] = __float_as_uint(a0);
        s[2 * k + 1] = __float_as_uint(a1);
    }
#pragma unroll
    for (int k = 0; k < BN / 2; ++k) {
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
    for (int c = 0; c < BN / 16; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t* e = s + 16 * c + 4 * q;
            acc[q] = f2_add(acc[q], f2_pack(__uint_as_float(e[0]), __uint_as_float(e[1])));
            acc[q] = f2_add(acc[q], f2_pack(__uint_as_float(e[2]), __uint_as_float(e[3])));
            pk[q] = e4m3x4(__uint_as_float(e[0]), __uint_as_float(e[1]), __uint_as_float(e[2]),
                           __uint_as_float(e[3]));
        }
        *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    const uint64_t t2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
    float r0, r1;
    f2_unpack(t2, r0, r1);
    return r0 + r1;
}

template <int D, int NKB, bool CAUSAL, bool QF>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p, const QParams qp) {
    using C = Cfg<D>;
    constexpr int kKeysPerBlk = BN / NKB;
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
    const int q_row0 = qt * (QT * BM);

    // key tiles each query tile visits: all of them, or (causal, bottom-right
    // aligned) up to the last key its last row sees; none for a tile wholly
    // past Lq
    int n_w[QT];
#pragma unroll
    for (int w = 0; w < QT; ++w) {
        int kv_end = p.Lk;
        if (CAUSAL) kv_end = max(0, min(kv_end, q_row0 + (w + 1) * BM + (p.Lk - p.Lq)));
        n_w[w] = q_row0 + w * BM < p.Lq ? (kv_end + BN - 1) / BN : 0;
    }
    const int n_max = max(n_w[0], n_w[1]);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            const bool four = (i >= C::kBarSEmpty && i < C::kBarSEmpty + QT) ||
                              (i >= C::kBarPFull && i < C::kBarPFull + QT) ||
                              (i >= C::kBarTok && i < C::kBarTok + QT);
            uint32_t cnt = four ? 4u : 1u;
            if (i == C::kBarQ && QF) cnt = 4u * QT;         // the softmax warps write Q
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    float* ks_s = reinterpret_cast<float*>(smem + C::kOffKs);
    float* vs_s = reinterpret_cast<float*>(smem + C::kOffVs);
    // launched as a programmatic dependent of the V quantisation: everything
    // above overlapped its tail; the quantised operands are read only below
    pdl_wait();
    {
        const float* ksrc = p.k_scale + (int64_t)bhk * p.nbk;
        const int nks = min(p.nbk, kKsSmem);
        for (int i = threadIdx.x; i < nks; i += kThreads) ks_s[i] = __ldg(&ksrc[i]);
        for (int i = threadIdx.x; i < D; i += kThreads) vs_s[i] = __ldg(&p.v_scale[(int64_t)bhk * D + i]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= kSoftWarps) {
      reg_dealloc<kProdRegs>();
      if (warp == kTmaWarp) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0 && n_max > 0) {
            if (!QF) tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            if (!QF) {
                mbar_arrive_expect_tx(&bars[C::kBarQ], QT * C::kQBytes);
                for (int w = 0; w < QT; ++w)
                    tma_load_2d(smem + C::kOffQ + w * C::kQBytes, &tmQ, &bars[C::kBarQ], 0,
                                bh * p.LpadQ + q_row0 + w * BM);
            }
            for (int t = 0; t < n_max; ++t) {
                const int s = t % C::kStages;
                const uint32_t ph = (t / C::kStages) & 1;
                if (!mbar_wait(&bars[C::kBarKEmpty + s], ph ^ 1, abort_flag, &g_attn_err, 1)) break;
                mbar_arrive_expect_tx(&bars[C::kBarKFull + s], C::kKBytes);
                tma_load_2d(smem + C::kOffK + s * C::kKBytes, &tmK, &bars[C::kBarKFull + s], 0,
                            bhk * p.LpadK + t * BN);
                if (!mbar_wait(&bars[C::kBarVEmpty + s], ph ^ 1, abort_flag, &g_attn_err, 2)) break;
                mbar_arrive_expect_tx(&bars[C::kBarVFull + s], C::kVBytes);
                tma_load_2d(smem + C::kOffV + s * C::kVBytes, &tmV, &bars[C::kBarVFull + s],
                            t * BN, bhk * D);
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0 && n_max > 0) {
            constexpr uint32_t kIdescQK = umma_idesc(2, 1, BM, BN);   // s8 x s8 -> s32
            constexpr uint32_t kIdescPV = umma_idesc(1, 0, BM, D);    // e4m3 x e4m3 -> f32
            const uint32_t sQ = smem_u32(smem + C::kOffQ);
            const uint32_t sK = smem_u32(smem + C::kOffK);
            const uint32_t sV = smem_u32(smem + C::kOffV);
            const uint32_t sP = smem_u32(smem + C::kOffP);

            // QK_w(t) for every query tile that visits key tile t. S_w holds
            // the 1.5 * 2^23 bias (written back by the softmax warps as they
            // release it); the MMA accumulates onto it.
            auto issue_qk = [&](int t) -> bool {
                const int s = t % C::kStages;
                const uint32_t ph = (t / C::kStages) & 1;
                if (!mbar_wait(&bars[C::kBarKFull + s], ph, abort_flag, &g_attn_err, 6)) return false;
                tc_fence_after();
                const uint64_t kdesc = umma_desc_kmajor(sK + s * C::kKBytes, D);
                for (int w = 0; w < QT; ++w) {
                    if (t >= n_w[w]) continue;
                    if (!mbar_wait(&bars[C::kBarSEmpty + w], t & 1, abort_flag, &g_attn_err, 7))
                        return false;
                    tc_fence_after();
                    const uint64_t qdesc = umma_desc_kmajor(sQ + w * C::kQBytes, D);
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk)
                        mma_i8_ss(tmem + w * BN, qdesc + 2 * kk, kdesc + 2 * kk, kIdescQK, 1u);
                    mma_commit(&bars[C::kBarSFull + w]);
                }
                mma_commit(&bars[C::kBarKEmpty + s]);
                return true;
            };
            // PV_w(t): O_w += P_w(t) V(t), once softmax w has written P_w(t)
            // and rescaled O_w for tile t (P_full).
            auto issue_pv = [&](int t) -> bool {
                const int s = t % C::kStages;
                const uint32_t ph = (t / C::kStages) & 1;
                if (!mbar_wait(&bars[C::kBarVFull + s], ph, abort_flag, &g_attn_err, 3)) return false;
                const uint64_t vdesc = umma_desc_kmajor(sV + s * C::kVBytes, 128);
                for (int w = 0; w < QT; ++w) {
                    if (t >= n_w[w]) continue;
                    if (!mbar_wait(&bars[C::kBarPFull + w], t & 1, abort_flag, &g_attn_err, 4))
                        return false;
                    tc_fence_after();
                    const uint64_t pdesc =
                        umma_desc_kmajor(sP + (w * C::kPBufs + (t & 1)) * C::kPBytes, 128);
#pragma unroll
                    for (int kk = 0; kk < BN / 32; ++kk)
                        mma_f8_ss(tmem + 256 + w * BM, pdesc + 2 * kk, vdesc + 2 * kk, kIdescPV,
                                  (t > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&bars[C::kBarODone + w]);
                }
                mma_commit(&bars[C::kBarVEmpty + s]);
                return true;
            };

            bool ok = mbar_wait(&bars[C::kBarQ], 0, abort_flag, &g_attn_err, 5);
            tc_fence_after();
            if (ok) ok = issue_qk(0);
            for (int t = 0; ok && t < n_max; ++t) {
                if (t + 1 < n_max) ok = issue_qk(t + 1);
                if (ok) ok = issue_pv(t);
            }
            // drain every MMA this thread issued before TMEM is released
            mma_commit(&bars[C::kBarFinal]);
            mbar_wait(&bars[C::kBarFinal], 0, abort_flag, &g_attn_err, 8);
        }
      }
    } else {
        reg_alloc<kSoftRegs>();
        // ---------------------------------------------------------- softmax
        // warp = query tile (w) x lane quarter (ww); the thread owns TMEM
        // lane 32 ww + lane: query row r of tile w, its 128 score columns and
        // its D output columns
        const int w = warp >> 2, ww = warp & 3;
        const int r = ww * 32 + lane;
        const int i = q_row0 + w * BM + r;
        const bool valid = i < p.Lq;
        const int n_t = n_w[w];
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(ww * 32) << 16);
        const uint32_t s_col = w * BN;
        const uint32_t o_col = 256 + w * BM;
        float qsc;
        if constexpr (QF) {
            // in-CTA Q: this thread's row is rotated and quantised with the
            // arithmetic of the Q/K quantisation kernel (same tile rows, same
            // block maxima), so the codes and scales are the same bits; the
            // codes go straight into the swizzled A operand of QK
            uint64_t x2[D / 2];
            {
                const uint16_t* src = qp.qbf + (bh / p.H) * qp.qs0 + (bh % p.H) * qp.qs1 + (int64_t)i * qp.qs2;
                if (qp.q_vec) {
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) {
                        const uint4 u = valid ? __ldg(reinterpret_cast<const uint4*>(src) + c) : make_uint4(0, 0, 0, 0);
                        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            x2[4 * c + e] = qrow::p2(qrow::bf16_bits_to_f32(wd[e] & 0xFFFFu), __uint_as_float(wd[e] & 0xFFFF0000u));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < D / 2; ++e) {
                        const uint32_t lo = valid ? __ldg(src + (int64_t)(2 * e) * qp.qs3) : 0u;
                        const uint32_t hi = valid ? __ldg(src + (int64_t)(2 * e + 1) * qp.qs3) : 0u;
                        x2[e] = qrow::p2(qrow::bf16_bits_to_f32(lo), qrow::bf16_bits_to_f32(hi));
                    }
                }
            }
            qrow::butterfly_pairs<D>(x2);
            float a = 0.0f;
#pragma unroll
            for (int j = 0; j < D / 2; ++j) a = fmax3(a, fabsf(qrow::p2lo(x2[j])), fabsf(qrow::p2hi(x2[j])));
            // a >= +0, so the bit patterns order like the values
            const unsigned am = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
            float* qmax = reinterpret_cast<float*>(smem + C::kOffQmax);
            if (lane == 0) qmax[warp] = __uint_as_float(am);
            asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");   // this tile's four warps
            const int wpb = p.blk_q >> 5, w0 = (ww / wpb) * wpb;        // warps of the row's block
            float amax = 0.0f;
            for (int k = w0; k < w0 + wpb; ++k) amax = fmaxf(amax, qmax[4 * w + k]);
            float sq = 0.0f, rr = 0.0f;
            if (amax != 0.0f) {
                sq = __fdiv_rn(amax, 127.0f);
                rr = __fdiv_rn(127.0f, amax);
            }
            uint8_t* qdst = smem + C::kOffQ + w * C::kQBytes + r * D;
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
                // 16-byte chunk c of the row at its 128B (D = 128) or 64B
                // (D = 64) swizzled position, as the TMA path would place it
                const int sc = D == 128 ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3));
                *reinterpret_cast<uint4*>(qdst + (sc << 4)) = qrow::row_codes16<D>(x2, rr, c);
            }
            fence_proxy_async_smem();              // read by the QK MMAs
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[C::kBarQ]);
            qsc = valid ? sq : 0.0f;
        } else {
            qsc = valid ? __ldg(&p.q_scale[(int64_t)bh * p.nbq + (i >> p.lg_blk_q)]) : 0.0f;
        }
        const float arow = qsc * p.logit_scale_log2;
        // last key this row sees (rows past Lq compute on zero padding and
        // are never written)
        int jlim = p.Lk - 1;
        if (CAUSAL && valid) jlim = min(jlim, i + (p.Lk - p.Lq));
        uint8_t* sPw = smem + C::kOffP + w * C::kPBufs * C::kPBytes;   // this tile's P buffers
        const float* ksrow = p.k_scale + (int64_t)bhk * p.nbk;

        // S_w starts as the bias 1.5 * 2^23 in every column: int32 accumulation
        // onto it leaves bits that read directly as the fp32 value 1.5 * 2^23 +
        // acc (exact, |acc| < 2^21)
        if (n_t > 0) {
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_fill32(lane_addr + s_col + 32 * c, kMagicI);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[C::kBarSEmpty + w]);
        }

        // tile 0 takes the first turn: tile 1 completes phase 0 of tok_0
        if (w == 1 && lane == 0) mbar_arrive(&bars[C::kBarTok + 0]);

        float m = -INFINITY, dsum = 0.0f;
        bool ok = true;
        for (int t = 0; t < n_t; ++t) {
            ok = warp_all(mbar_wait(&bars[C::kBarSFull + w], t & 1, abort_flag, &g_attn_err, 9));
            if (!ok) break;
            tc_fence_after();
            // the whole score row into registers, then S goes back to the MMA
            // warp with the bias rewritten for tile t + 1
            uint32_t s[BN];
            tmem_ld128(lane_addr + s_col, s);
            tmem_wait_ld128(s);
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_fill32(lane_addr + s_col + 32 * c, kMagicI);

            const int j0 = t * BN;
            // a tile that reaches past some row's last visible key needs masking
            const bool need_mask = __any_sync(0xffffffffu, j0 + BN - 1 > jlim);
            float kc[NKB];
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) {
                const int bi = min((j0 + kb * kKeysPerBlk) >> p.lg_blk_k, p.nbk - 1);
                kc[kb] = (bi < kKsSmem ? ks_s[bi] : __ldg(&ksrow[bi])) * arow;
            }
            // QK and update_mdo (max part). y = acc * kc is monotonic in acc
            // (kc >= 0), so each K block's max is taken on the raw biased
            // values (three-input max), then unbiased and scaled.
            float mt = -INFINITY;
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) {
                const float cm = need_mask
                    ? block_max<kKeysPerBlk, true>(s + kb * kKeysPerBlk, j0 + kb * kKeysPerBlk, jlim)
                    : block_max<kKeysPerBlk, false>(s + kb * kKeysPerBlk, j0 + kb * kKeysPerBlk, jlim);
                if (cm != -INFINITY) mt = fmaxf(mt, (cm - kMagicF) * kc[kb]);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[C::kBarSEmpty + w]);
            const float m_new = fmaxf(m, mt);
            const float msub = (m_new == -INFINITY) ? 0.0f : m_new;
            const float alpha = ex2_approx(m - msub);
            // the exponentials of the two query tiles take turns (token tok_w,
            // passed on below), so one tile's max and rescale overlap the
            // other's MUFU work instead of both tiles contending for it
            ok = warp_all(mbar_wait(&bars[C::kBarTok + w], t & 1, abort_flag, &g_attn_err, 12));
            if (!ok) break;

            // accumulate_d and RS_32_to_8: p448 = 448 * 2^(y - m') =
            // 2^(acc * kc + log2(448) - m'), one FMA per key (f32x2). Each
            // 32-key chunk of P8 goes to shared memory in the 128B-swizzled
            // K-major layout (16-byte chunk c of row r at c ^ (r & 7)). Buffer
            // t & 1 was last read by PV(t - 2), awaited before tile t - 1's
            // rescale.
            uint8_t* prow = sPw + (t & 1) * C::kPBytes + r * 128;
            const float tsum = need_mask ? row_exp<NKB, true>(s, kc, kLog2_448 - msub, j0, jlim, prow, r)
                                         : row_exp<NKB, false>(s, kc, kLog2_448 - msub, j0, jlim, prow, r);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[C::kBarTok + (w ^ 1)]);
            dsum = dsum * alpha + tsum;
            if (t > 0) {
                // update_mdo (rescale part): PV(t-1) must have landed in O first;
                // then O *= alpha, skipped when no row of the warp changed its max
                ok = warp_all(mbar_wait(&bars[C::kBarODone + w], (t - 1) & 1, abort_flag,
                                        &g_attn_err, 10));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.0f)) {
                    const uint64_t al2 = f2_pack(alpha, alpha);
#pragma unroll
                    for (int c2 = 0; c2 < D / 64; ++c2) {
                        uint32_t o[64];
                        tmem_ld32(lane_addr + o_col + 64 * c2, slice32(o));
                        tmem_ld32(lane_addr + o_col + 64 * c2 + 32, slice32(o + 32));
                        tmem_wait_ld(slice32(o));
                        tmem_wait_ld(slice32(o + 32));
#pragma unroll
                        for (int e = 0; e < 64; e += 2) {
                            float a0, a1;
                            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2),
                                      a0, a1);
                            o[e] = __float_as_uint(a0);
                            o[e + 1] = __float_as_uint(a1);
                        }
                        tmem_st32(lane_addr + o_col + 64 * c2, slice32(o));
                        tmem_st32(lane_addr + o_col + 64 * c2 + 32, slice32(o + 32));
                    }
                    tmem_wait_st();
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[C::kBarPFull + w]);
            m = m_new;
        }
        // the other tile may visit more key tiles (causal, or this tile lies
        // past Lq): keep passing the turn until it is done
        for (int t = n_t; ok && t < n_w[w ^ 1]; ++t) {
            ok = warp_all(mbar_wait(&bars[C::kBarTok + w], t & 1, abort_flag, &g_attn_err, 13));
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(&bars[C::kBarTok + (w ^ 1)]);
        }

        // epilogue: out = O * v_scale / (448 d) -> bf16 (448 is inside the
        // exponent), caller's strides
        __nv_bfloat16* orow = p.out + b * p.os0 + h * p.os1 + (int64_t)i * p.os2;
        if (ok && n_t > 0) {
            ok = warp_all(mbar_wait(&bars[C::kBarODone + w], (n_t - 1) & 1, abort_flag,
                                    &g_attn_err, 11));
            if (ok) {
                tc_fence_after();
                const float inv = dsum > 0.0f ? 1.0f / dsum : 0.0f;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(lane_addr + o_col + 32 * c, o);
                    tmem_wait_ld(o);
                    if (valid) {
                        uint32_t packed[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 vs2 = *reinterpret_cast<const float2*>(vs_s + 32 * c + e);
                            const float v0 = __uint_as_float(o[e]) * (vs2.x * inv);
                            const float v1 = __uint_as_float(o[e + 1]) * (vs2.y * inv);
                            const __nv_bfloat162 pr = __floats2bfloat162_rn(v0, v1);
                            packed[e / 2] = *reinterpret_cast<const uint32_t*>(&pr);
                        }
                        if (p.out_vec) {
                            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                dst[q4] = make_uint4(packed[4 * q4], packed[4 * q4 + 1],
                                                     packed[4 * q4 + 2], packed[4 * q4 + 3]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const uint16_t bits16 = (e & 1) ? (packed[e / 2] >> 16) : (packed[e / 2] & 0xFFFFu);
                                *reinterpret_cast<uint16_t*>(orow + (int64_t)(32 * c + e) * p.os3) = bits16;
                            }
                        }
                    }
                }
            }
        } else if (n_t == 0 && valid) {
            for (int d = 0; d < D; ++d) orow[(int64_t)d * p.os3] = __float2bfloat16_rn(0.0f);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D uint8 tensor map: `rows` rows of `cols` bytes (row pitch = cols), box
// {box_cols, box_rows}, swizzle matching the row length of the box.
bool encode_u8_2d(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows,
                  uint32_t box_cols, uint32_t box_rows) {
    auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw =
        box_cols == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NKB, bool CAUSAL>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const Params& p, const QParams& qp, bool qfused, dim3 grid, cudaStream_t s) {
    auto kern = qfused ? attn_fwd_kernel<D, NKB, CAUSAL, true> : attn_fwd_kernel<D, NKB, CAUSAL, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg<D>::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, grid, dim3(kThreads), Cfg<D>::kSmemBytes, s, tq, tk, tv, p, qp);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, int NKB>
cudaError_t launch_c(bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, const Params& p, const QParams& qp, bool qfused,
                     dim3 grid, cudaStream_t s) {
    return causal ? launch_t<D, NKB, true>(tq, tk, tv, p, qp, qfused, grid, s)
                  : launch_t<D, NKB, false>(tq, tk, tv, p, qp, qfused, grid, s);
}

template <int D>
cudaError_t launch_d(int nkb, bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, const Params& p, const QParams& qp, bool qfused,
                     dim3 grid, cudaStream_t s) {
    switch (nkb) {
        case 1: return launch_c<D, 1>(causal, tq, tk, tv, p, qp, qfused, grid, s);
        case 2: return launch_c<D, 2>(causal, tq, tk, tv, p, qp, qfused, grid, s);
        default: return launch_c<D, 4>(causal, tq, tk, tv, p, qp, qfused, grid, s);
    }
}

}  // namespace

cudaError_t launch_attn_fwd(const AttnArgs& a, cudaStream_t s) {
    const int LpadQ = static_cast<int>(round_up(a.Lq, kTile));
    const int LpadK = static_cast<int>(round_up(a.Lk, kTile));
    CUtensorMap tq, tk, tv;
    memset(&tq, 0, sizeof tq);                     // not read by the in-CTA Q path
    if ((!a.qfused && !encode_u8_2d(&tq, a.q8, a.D, (uint64_t)a.B * a.H * LpadQ, a.D, BM)) ||
        !encode_u8_2d(&tk, a.k8, a.D, (uint64_t)a.B * a.Hk * LpadK, a.D, BN) ||
        !encode_u8_2d(&tv, a.v8t, LpadK, (uint64_t)a.B * a.Hk * a.D, BN, a.D))
        return cudaErrorInvalidValue;
    Params p;
    p.q_scale = a.q_scale;
    p.k_scale = a.k_scale;
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
    p.blk_q = a.blk_q;
    p.blk_k = a.blk_k;
    p.nbq = static_cast<int>(ceil_div(a.Lq, a.blk_q));
    p.nbk = static_cast<int>(ceil_div(a.Lk, a.blk_k));
    p.lg_blk_q = __builtin_ctz(static_cast<unsigned>(a.blk_q));
    p.lg_blk_k = __builtin_ctz(static_cast<unsigned>(a.blk_k));
    p.logit_scale_log2 = a.softmax_scale / static_cast<float>(a.D) * kLog2e;
    p.heavy_first = a.causal ? 1 : 0;
    p.out_vec = (a.out_stride[3] == 1 && a.out_stride[0] % 8 == 0 && a.out_stride[1] % 8 == 0 &&
                 a.out_stride[2] % 8 == 0 && reinterpret_cast<uintptr_t>(a.out) % 16 == 0)
                    ? 1
                    : 0;
    QParams qp;
    qp.qbf = static_cast<const uint16_t*>(a.q16.ptr);
    qp.qs0 = a.q16.stride[0];
    qp.qs1 = a.q16.stride[1];
    qp.qs2 = a.q16.stride[2];
    qp.qs3 = a.q16.stride[3];
    qp.q_vec = (a.qfused && a.q16.stride[3] == 1 && a.q16.stride[0] % 8 == 0 && a.q16.stride[1] % 8 == 0 &&
               a.q16.stride[2] % 8 == 0 && reinterpret_cast<uintptr_t>(a.q16.ptr) % 16 == 0)
                  ? 1
                  : 0;
    const int nqt = static_cast<int>(ceil_div(a.Lq, QT * BM));
    const dim3 grid = a.causal ? dim3(a.B * a.H, nqt) : dim3(nqt, a.B * a.H);
    const int nkb = BN / a.blk_k;
    return a.D == 128 ? launch_d<128>(nkb, a.causal != 0, tq, tk, tv, p, qp, a.qfused != 0, grid, s)
                      : launch_d<64>(nkb, a.causal != 0, tq, tk, tv, p, qp, a.qfused != 0, grid, s);
}

unsigned read_clear_attn_error() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_err, sizeof v) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_attn_err, &zero, sizeof zero);
    return v;
}

}  // namespace sage
