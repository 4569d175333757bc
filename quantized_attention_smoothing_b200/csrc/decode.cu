// decode.cu -- paged FP8-KV decode with MTP query tokens, GQA and a sliding
// window ("[FlyDSL] [Misc] pa_decode: key the tile kernel on FlyDSL dtypes
// and drop the batch-first plan grid": window-family workload with per-token
// FP8 K/V scales, MTP4, GQA16, one KV head, page 128; Changes: Q/P quantised
// to the FP8 format of the cache (Q here), PV on bf16 operands because a
// per-token V scale cannot be factored out of the sum).
//
// Split-KV. decode_split_kernel: CTA (split, b * Hk + hk), 8 warps, handles
// up to 512 consecutive keys of the union of the T query tokens' windows for
// all R = T * (H / Hk) query rows of kv head hk. Two warpgroups take
// alternate 64-key chunks (16 rows per warp) with their own running softmax
// state, merged at the end:
//   0. the keys' cache rows are looked up through the page table (page ids
//      bounds-checked) and every K row, V row and per-token scale of the
//      split is requested at once with cp.async, one commit group per
//      64-key chunk;
//   1. while those land, the Q rows are rotated and quantised: bf16 -> fp32
//      butterfly (two threads per row, the last stage across the pair by
//      shuffles) -> e4m3 with scale max|q_hat| / 448 (the fp32 operations
//      of the quantisation kernels);
//   2. per 64-key chunk, once its copies have landed: V decoded exactly to
//      bf16; S = Q8 K8^T with e4m3 mma.sync (fp32 accumulate), scaled by
//      s_q * s_k * softmax_scale / D, masked to each row's own window (no
//      per-key test for chunks inside every row's window);
//      online softmax in base 2; P' = p * s_v rounded to bf16; O += P' V with
//      bf16 mma.sync;
//   3. the second warpgroup's (m, l, O) merged into the first's, then to the
//      workspace.
// decode_combine_kernel merges the splits (log-sum-exp) and writes bf16
// through the caller's strides.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {
namespace {

__device__ unsigned g_decode_err;
constexpr unsigned kErrDecodeRange = 2u;     // ctx or page id out of range (clamped)

constexpr int kD = 128;
constexpr int kSplit = 512;                  // keys per CTA
constexpr int kChunk = 64;                   // keys per inner step
constexpr int kNChunk = kSplit / kChunk;     // 64-key chunks per CTA
constexpr int kDecThreads = 256;             // two warpgroups of 4 warps
constexpr int kMaxRows = 64;                 // T * (H / Hk)
constexpr int kKPitch = kD + 16;             // bytes per K row in smem
constexpr int kVPitch = kD + 8;              // bf16 elements per V row in smem
constexpr float kLog2e = 1.4426950408889634f;

// dynamic shared memory of decode_split_kernel
struct DecSmem {
    static constexpr int kOffK = 0;                                   // [kSplit][kKPitch] e4m3
    static constexpr int kOffV = kOffK + kSplit * kKPitch;            // [kSplit][kD] e4m3
    static constexpr int kOffVbf = kOffV + kSplit * kD;               // [2][kChunk][kVPitch] bf16
    static constexpr int kOffQ = kOffVbf + 2 * kChunk * kVPitch * 2;  // [kMaxRows][kD] e4m3
    static constexpr int kOffKs = kOffQ + kMaxRows * kD;              // [kSplit] fp32
    static constexpr int kOffVs = kOffKs + kSplit * 4;                // [kSplit] fp32
    static constexpr int kOffTok = kOffVs + kSplit * 4;               // [kSplit] int64 (-1: none)
    static constexpr int kOffSq = kOffTok + kSplit * 8;               // [kMaxRows] fp32
    static constexpr int kOffBad = kOffSq + kMaxRows * 4;             // [kNChunk] int
    static constexpr int kBytes = kOffBad + kNChunk * 4;
    // merge area of the second warpgroup's state, over the K rows (read by then)
    static constexpr int kMergeBytes = 4 * 32 * (64 + 4) * 4;
    static_assert(kMergeBytes <= kSplit * kKPitch, "merge area");
    static_assert(kBytes <= 227 * 1024, "shared memory");
};

struct DecParams {
    const uint16_t* q;
    int64_t qs0, qs1, qs2, qs3;              // q strides [B, T, H, D] (elements)
    const uint8_t* kc;
    const uint8_t* vc;
    const float* ksc;
    const float* vsc;
    const int32_t* ptab;
    const int32_t* ctx;
    int T, H, Hk, G, R, Rpad, page, max_pages, num_pages, window, nsplit;
    int q_vec;                               // q rows contiguous and 16-byte aligned
    float logit_scale_log2;                  // softmax_scale / D * log2(e)
    float* part;                             // [B*Hk][nsplit][Rpad][D + 2]
    __nv_bfloat16* out;
    int64_t os0, os1, os2, os3;
};

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t r;
    const uint16_t in = static_cast<uint16_t>(code);
    asm("{\n\t.reg .b32 h2;\n\tcvt.rn.f16x2.e4m3x2 h2, %1;\n\tmov.b32 %0, h2;\n\t}" : "=r"(r) : "h"(in));
    return __half2float(__ushort_as_half(static_cast<uint16_t>(r & 0xFFFFu)));
}

// four e4m3 bytes -> two packed bf16 pairs (exact: e4m3 values are bf16 values)
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
    uint32_t h01, h23;
    const uint16_t w01 = static_cast<uint16_t>(w & 0xFFFFu), w23 = static_cast<uint16_t>(w >> 16);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"(w01));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"(w23));
    const __half2 a = *reinterpret_cast<const __half2*>(&h01);
    const __half2 b = *reinterpret_cast<const __half2*>(&h23);
    const __nv_bfloat162 ab = __floats2bfloat162_rn(__low2float(a), __high2float(a));
    const __nv_bfloat162 bb = __floats2bfloat162_rn(__low2float(b), __high2float(b));
    lo = *reinterpret_cast<const uint32_t*>(&ab);
    hi = *reinterpret_cast<const uint32_t*>(&bb);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    const uint32_t d = smem_u32(dst);
    const int n = valid ? 16 : 0;                 // 0 bytes read -> zero fill
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
    const uint32_t d = smem_u32(dst);
    const int n = valid ? 4 : 0;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Wait until at most `pending` (0 .. 3) of this thread's commit groups are
// outstanding.
__device__ __forceinline__ void cp_async_wait_pending(int pending) {
    switch (pending) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    }
}
static_assert(kNChunk == 8, "each warpgroup commits 4 chunk groups");

// Barrier of one warpgroup (named barrier 1 + grp, 128 threads).
__device__ __forceinline__ void group_sync(int grp) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + grp) : "memory");
}

__device__ __forceinline__ void mma_e4m3_16832(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* row_addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(row_addr)));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecParams p) {
    extern __shared__ __align__(128) uint8_t dsm[];
    uint8_t (*ks8)[kKPitch] = reinterpret_cast<uint8_t (*)[kKPitch]>(dsm + DecSmem::kOffK);
    uint8_t (*vs8)[kD] = reinterpret_cast<uint8_t (*)[kD]>(dsm + DecSmem::kOffV);
    __nv_bfloat16 (*vbf)[kVPitch] = reinterpret_cast<__nv_bfloat16 (*)[kVPitch]>(dsm + DecSmem::kOffVbf);
    uint8_t (*q8s)[kD] = reinterpret_cast<uint8_t (*)[kD]>(dsm + DecSmem::kOffQ);
    float* kscl = reinterpret_cast<float*>(dsm + DecSmem::kOffKs);
    float* vscl = reinterpret_cast<float*>(dsm + DecSmem::kOffVs);
    int64_t* tokr = reinterpret_cast<int64_t*>(dsm + DecSmem::kOffTok);
    float* sq = reinterpret_cast<float*>(dsm + DecSmem::kOffSq);
    int* chunk_bad = reinterpret_cast<int*>(dsm + DecSmem::kOffBad);

    const int split = blockIdx.x, bhk = blockIdx.y;
    const int b = bhk / p.Hk, hk = bhk % p.Hk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tg = lane & 3;
    const int grp = warp >> 2, gtid = tid & 127;     // warpgroup, thread within it

    int ctx = p.ctx[b];
    const int cap = p.max_pages * p.page;
    if (ctx > cap || ctx < 0) {
        if (tid == 0 && split == 0) atomicCAS(&g_decode_err, 0u, kErrDecodeRange);
        ctx = max(0, min(ctx, cap));
    }
    const int lo = max(0, ctx - p.T - p.window + 1);
    const int k_begin = lo + split * kSplit;
    const int k_end = min(ctx, k_begin + kSplit);      // exclusive
    const int nk = max(0, k_end - k_begin);

    // ---- 0. cache rows of this split's keys, then every K / V row and
    // per-token scale requested at once; warpgroup grp requests the chunks it
    // will process (c = grp, grp + 2, ...), one commit group per chunk
    if (tid < kNChunk) chunk_bad[tid] = 0;
    __syncthreads();
    for (int kr = tid; kr < kSplit; kr += kDecThreads) {
        int64_t tok = -1;
        if (kr < nk) {
            const int j = k_begin + kr;
            const int pg = __ldg(&p.ptab[(int64_t)b * p.max_pages + j / p.page]);
            if (pg < 0 || pg >= p.num_pages) {
                atomicCAS(&g_decode_err, 0u, kErrDecodeRange);
                atomicOr(&chunk_bad[kr / kChunk], 1);
            } else {
                tok = ((int64_t)pg * p.Hk + hk) * p.page + (j % p.page);
            }
        }
        tokr[kr] = tok;
    }
    __syncthreads();
    for (int c = grp; c < kNChunk; c += 2) {
        // 64 keys x (8 K pieces + 8 V pieces) of 16 bytes; two scales per key
        for (int i = gtid; i < kChunk * 16; i += 128) {
            const int kr = c * kChunk + i / 16, piece = i % 16;
            const int64_t tok = tokr[kr];
            const bool ok = tok >= 0;
            const int64_t off = ok ? tok * kD + (piece & 7) * 16 : 0;
            if (piece < 8) cp_async16(&ks8[kr][piece * 16], p.kc + off, ok);
            else cp_async16(&vs8[kr][(piece - 8) * 16], p.vc + off, ok);
        }
        {
            const int kr = c * kChunk + (gtid & (kChunk - 1));
            const int64_t tok = tokr[kr];
            if (gtid < kChunk) cp_async4(&kscl[kr], p.ksc + (tok >= 0 ? tok : 0), tok >= 0);
            else cp_async4(&vscl[kr], p.vsc + (tok >= 0 ? tok : 0), tok >= 0);
        }
        cp_async_commit();
    }

    // ---- 1. query rows: rotate and quantise to e4m3, two threads per row
    // (thread half hq holds elements [64 hq, 64 hq + 64)). Every thread runs
    // the whole sequence, shuffles included; rows past R load zeros, which
    // gives them zero codes and a zero scale.
    if (grp == 0) {
        const int r = tid >> 1, hq = tid & 1;
        const bool rv = r < p.R;
        const int t = rv ? r / p.G : 0, h = rv ? hk * p.G + r % p.G : 0;
        const uint16_t* src = p.q + b * p.qs0 + t * p.qs1 + h * p.qs2 + (int64_t)(hq * 64) * p.qs3;
        float x[64];
        if (p.q_vec) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 u = rv ? __ldg(reinterpret_cast<const uint4*>(src) + c) : make_uint4(0, 0, 0, 0);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * c + 2 * e] = __uint_as_float(w[e] << 16);
                    x[8 * c + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                }
            }
        } else {
#pragma unroll
            for (int d = 0; d < 64; ++d)
                x[d] = rv ? __uint_as_float(static_cast<uint32_t>(__ldg(src + d * p.qs3)) << 16) : 0.0f;
        }
        // stages h = 1 .. 32 inside the half
#pragma unroll
        for (int lg = 0; lg < 6; ++lg) {
            const int hh = 1 << lg;
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) {
                const int j = ((kk >> lg) << (lg + 1)) + (kk & (hh - 1));
                const float a = x[j], c = x[j + hh];
                x[j] = __fadd_rn(a, c);
                x[j + hh] = __fsub_rn(a, c);
            }
        }
        // stage h = 64 across the pair: x[j] +- x[j + 64]
#pragma unroll
        for (int j = 0; j < 64; ++j) {
            const float y = __shfl_xor_sync(0xffffffffu, x[j], 1);
            x[j] = hq == 0 ? __fadd_rn(x[j], y) : __fsub_rn(y, x[j]);
        }
        float amax = 0.0f;
#pragma unroll
        for (int d = 0; d < 64; ++d) amax = fmaxf(amax, fabsf(x[d]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        float s = 0.0f, rr = 0.0f;
        if (amax != 0.0f) {
            s = __fdiv_rn(amax, 448.0f);
            rr = __fdiv_rn(448.0f, amax);
        }
        if (hq == 0) sq[r] = s;
#pragma unroll
        for (int d = 0; d < 64; d += 16) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t lo16 = e4m3x2_rn_satfinite(__fmul_rn(x[d + 4 * e], rr), __fmul_rn(x[d + 4 * e + 1], rr));
                const uint32_t hi16 = e4m3x2_rn_satfinite(__fmul_rn(x[d + 4 * e + 2], rr), __fmul_rn(x[d + 4 * e + 3], rr));
                w4[e] = lo16 | (hi16 << 16);
            }
            *reinterpret_cast<uint4*>(&q8s[r][hq * 64 + d]) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
    __syncthreads();

    // A fragments of this warp's 16 rows (4 k-steps of 32 channels), kept in registers
    const int row0 = (warp & 3) * 16;
    uint32_t qa[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        qa[kk][0] = *reinterpret_cast<const uint32_t*>(&q8s[row0 + g][kk * 32 + tg * 4]);
        qa[kk][1] = *reinterpret_cast<const uint32_t*>(&q8s[row0 + g + 8][kk * 32 + tg * 4]);
        qa[kk][2] = *reinterpret_cast<const uint32_t*>(&q8s[row0 + g][kk * 32 + 16 + tg * 4]);
        qa[kk][3] = *reinterpret_cast<const uint32_t*>(&q8s[row0 + g + 8][kk * 32 + 16 + tg * 4]);
    }
    // per-thread rows: ra = row0 + g, rb = row0 + g + 8
    const int ra = row0 + g, rb = ra + 8;
    const bool va = ra < p.R, vb_ = rb < p.R;
    const int pa = va ? ctx - p.T + ra / p.G : -1;      // query position of each row
    const int pb = vb_ ? ctx - p.T + rb / p.G : -1;
    const float ca = va ? sq[ra] * p.logit_scale_log2 : 0.0f;
    const float cb = vb_ ? sq[rb] * p.logit_scale_log2 : 0.0f;

    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;

    const int nchunks = (nk + kChunk - 1) / kChunk;
    __nv_bfloat16 (*vb)[kVPitch] = vbf + grp * kChunk;   // this warpgroup's bf16 V chunk
    for (int ci = 0; grp + 2 * ci < nchunks; ++ci) {
        const int c = grp + 2 * ci;
        const int c0 = c * kChunk;                      // chunk's first key, split-relative
        cp_async_wait_pending(kNChunk / 2 - 1 - ci);   // this thread's copies of chunk c are in
        group_sync(grp);                                // the group's; its previous vb reads done
        // V e4m3 -> bf16 (exact)
        for (int i = gtid; i < kChunk * (kD / 4); i += 128) {
            const int kr = i / (kD / 4), c4 = (i % (kD / 4)) * 4;
            uint32_t lo2, hi2;
            e4m3x4_to_bf16x4(*reinterpret_cast<const uint32_t*>(&vs8[c0 + kr][c4]), lo2, hi2);
            *reinterpret_cast<uint2*>(&vb[kr][c4]) = make_uint2(lo2, hi2);
        }
        group_sync(grp);
        // keys [jf, jf + 64) inside every row's window and all present: no
        // per-key tests
        const int jf = k_begin + c0;
        const bool full = c0 + kChunk <= nk && !chunk_bad[c] && jf + kChunk - 1 <= ctx - p.T &&
                          jf > ctx - 1 - p.window;

        // ---- 2b. S = Q8 K8^T for 64 keys (8 n-tiles of 8 keys)
        float sacc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.0f;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&ks8[c0 + nt * 8 + g][kk * 32 + tg * 4]);
                const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&ks8[c0 + nt * 8 + g][kk * 32 + 16 + tg * 4]);
                mma_e4m3_16832(sacc[nt], qa[kk], b0, b1);
            }
        }
        // scale, mask to each row's window, base-2 logits
        float mx_a = -INFINITY, mx_b = -INFINITY;
        if (full) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float ksv = kscl[c0 + nt * 8 + tg * 2 + e];
                    sacc[nt][e] = sacc[nt][e] * ca * ksv;
                    sacc[nt][2 + e] = sacc[nt][2 + e] * cb * ksv;
                    mx_a = fmaxf(mx_a, sacc[nt][e]);
                    mx_b = fmaxf(mx_b, sacc[nt][2 + e]);
                }
            // rows past R: logits are 0 * ..., masked here as before
            if (!va) mx_a = -INFINITY;
            if (!vb_) mx_b = -INFINITY;
            if (!va || !vb_) {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    if (!va) sacc[nt][0] = sacc[nt][1] = -INFINITY;
                    if (!vb_) sacc[nt][2] = sacc[nt][3] = -INFINITY;
                }
            }
        } else {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int kr = c0 + nt * 8 + tg * 2 + e;
                    const int j = k_begin + kr;
                    const float ksv = kscl[kr];
                    const bool okk = kr < nk && tokr[kr] >= 0;
                    const bool vis_a = okk && j <= pa && j > pa - p.window;
                    const bool vis_b = okk && j <= pb && j > pb - p.window;
                    sacc[nt][e] = vis_a ? sacc[nt][e] * ca * ksv : -INFINITY;
                    sacc[nt][2 + e] = vis_b ? sacc[nt][2 + e] * cb * ksv : -INFINITY;
                    mx_a = fmaxf(mx_a, sacc[nt][e]);
                    mx_b = fmaxf(mx_b, sacc[nt][2 + e]);
                }
        }
#pragma unroll
        for (int o2 = 1; o2 <= 2; o2 <<= 1) {
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, o2));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, o2));
        }
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const float sub_a = mn_a == -INFINITY ? 0.0f : mn_a;
        const float sub_b = mn_b == -INFINITY ? 0.0f : mn_b;
        const float al_a = ex2_approx(m_a - sub_a), al_b = ex2_approx(m_b - sub_b);
        // P' = p * s_v (bf16) as A fragments of the PV mma (two n-tiles = 16 keys)
        uint32_t pa_frag[4][4];
        float ls_a = 0.0f, ls_b = 0.0f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kr = c0 + nt * 8 + tg * 2 + e;
                const float pa_ = ex2_approx(sacc[nt][e] - sub_a);
                const float pb_ = ex2_approx(sacc[nt][2 + e] - sub_b);
                ls_a += pa_;
                ls_b += pb_;
                pv[e] = pa_ * vscl[kr];
                pv[2 + e] = pb_ * vscl[kr];
            }
            const int ks = nt >> 1, half = nt & 1;
            pa_frag[ks][half * 2 + 0] = pack_bf16(pv[0], pv[1]);     // row g
            pa_frag[ks][half * 2 + 1] = pack_bf16(pv[2], pv[3]);     // row g + 8
        }
#pragma unroll
        for (int o2 = 1; o2 <= 2; o2 <<= 1) {
            ls_a += __shfl_xor_sync(0xffffffffu, ls_a, o2);
            ls_b += __shfl_xor_sync(0xffffffffu, ls_b, o2);
        }
        l_a = l_a * al_a + ls_a;
        l_b = l_b * al_b + ls_b;
        m_a = mn_a;
        m_b = mn_b;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            o[n][0] *= al_a;
            o[n][1] *= al_a;
            o[n][2] *= al_b;
            o[n][3] *= al_b;
        }
        // ---- 2c. O += P' V (4 k-steps of 16 keys x 16 n-tiles of 8 channels)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            // A fragment layout of m16n8k16: {row g: k 0-7 pair, row g+8: k 0-7 pair,
            // row g: k 8-15 pair, row g+8: k 8-15 pair}
            const uint32_t afr[4] = {pa_frag[ks][0], pa_frag[ks][1], pa_frag[ks][2], pa_frag[ks][3]};
#pragma unroll
            for (int np = 0; np < 8; ++np) {        // pairs of n-tiles
                // lanes 0-15 address keys ks*16 + (lane & 15) of n-tile 2np,
                // lanes 16-31 the same keys of n-tile 2np + 1
                const int krow = ks * 16 + (lane & 15);
                const int col = (2 * np + (lane >> 4)) * 8;
                uint32_t bfr[4];
                ldmatrix_x4_trans(bfr, &vb[krow][col]);
                mma_bf16_16816(o[2 * np], afr, bfr[0], bfr[1]);
                mma_bf16_16816(o[2 * np + 1], afr, bfr[2], bfr[3]);
            }
        }
    }
    cp_async_wait_pending(0);       // no copy may outlive the CTA

    // ---- 3. merge the second warpgroup's state into the first's, over the
    // K rows (every read of them is done after this barrier)
    __syncthreads();
    float* mg = reinterpret_cast<float*>(dsm + DecSmem::kOffK) + ((warp & 3) * 32 + lane) * (64 + 4);
    if (grp == 1) {
#pragma unroll
        for (int n = 0; n < 16; ++n)
            *reinterpret_cast<float4*>(mg + 4 * n) = make_float4(o[n][0], o[n][1], o[n][2], o[n][3]);
        *reinterpret_cast<float4*>(mg + 64) = make_float4(m_a, m_b, l_a, l_b);
    }
    __syncthreads();
    if (grp == 1) return;
    {
        const float4 st = *reinterpret_cast<const float4*>(mg + 64);
        const float Ma = fmaxf(m_a, st.x), Mb = fmaxf(m_b, st.y);
        const float w0a = m_a == -INFINITY ? 0.0f : ex2_approx(m_a - Ma);
        const float w1a = st.x == -INFINITY ? 0.0f : ex2_approx(st.x - Ma);
        const float w0b = m_b == -INFINITY ? 0.0f : ex2_approx(m_b - Mb);
        const float w1b = st.y == -INFINITY ? 0.0f : ex2_approx(st.y - Mb);
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            const float4 o1 = *reinterpret_cast<const float4*>(mg + 4 * n);
            o[n][0] = o[n][0] * w0a + o1.x * w1a;
            o[n][1] = o[n][1] * w0a + o1.y * w1a;
            o[n][2] = o[n][2] * w0b + o1.z * w1b;
            o[n][3] = o[n][3] * w0b + o1.w * w1b;
        }
        l_a = l_a * w0a + st.z * w1a;
        l_b = l_b * w0b + st.w * w1b;
        m_a = Ma;
        m_b = Mb;
    }

    // partial results of this split
    // (rows beyond Rpad exist only as padding of the 4 x 16 row grid)
    if (row0 < p.Rpad) {
        const int64_t base = ((int64_t)bhk * p.nsplit + split) * p.Rpad;
        float* rowa = p.part + (base + ra) * (kD + 2);
        float* rowb = p.part + (base + rb) * (kD + 2);
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            *reinterpret_cast<float2*>(rowa + n * 8 + tg * 2) = make_float2(o[n][0], o[n][1]);
            *reinterpret_cast<float2*>(rowb + n * 8 + tg * 2) = make_float2(o[n][2], o[n][3]);
        }
        if (tg == 0) {
            rowa[kD] = m_a;
            rowa[kD + 1] = l_a;
            rowb[kD] = m_b;
            rowb[kD + 1] = l_b;
        }
    }
}

// One CTA per (row, b * hk), one thread per channel: merges the splits of
// the row (log-sum-exp rescaling) and writes bf16.
__global__ void __launch_bounds__(kD) decode_combine_kernel(const DecParams p) {
    const int r = blockIdx.x, bhk = blockIdx.y;
    const int b = bhk / p.Hk, hk = bhk % p.Hk;
    const int d = threadIdx.x;
    const int t = r / p.G, h = hk * p.G + r % p.G;
    const int64_t stride = (int64_t)p.Rpad * (kD + 2);
    const float* row0 = p.part + ((int64_t)bhk * p.nsplit * p.Rpad + r) * (kD + 2);
    float M = -INFINITY;
#pragma unroll 4
    for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, __ldg(row0 + s * stride + kD));
    float acc = 0.0f, den = 0.0f;
    if (M != -INFINITY) {
#pragma unroll 4
        for (int s = 0; s < p.nsplit; ++s) {
            const float* row = row0 + s * stride;
            const float ms = __ldg(row + kD);
            const float w = (ms == -INFINITY) ? 0.0f : ex2_approx(ms - M);
            acc = fmaf(w, __ldg(row + d), acc);
            den = fmaf(w, __ldg(row + kD + 1), den);
        }
    }
    const float y = den > 0.0f ? acc / den : 0.0f;
    p.out[b * p.os0 + t * p.os1 + h * p.os2 + (int64_t)d * p.os3] = __float2bfloat16_rn(y);
}

int nsplit_for(int T, int window) {
    return static_cast<int>(ceil_div(window + T - 1, kSplit));
}

}  // namespace

size_t decode_ws_bytes(int B, int T, int H, int Hk, int D, int window) {
    const int R = T * (H / Hk);
    const int Rpad = static_cast<int>(round_up(R, 16));
    return (size_t)B * Hk * nsplit_for(T, window) * Rpad * (D + 2) * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    DecParams p;
    p.q = static_cast<const uint16_t*>(a.q.ptr);
    p.qs0 = a.q.stride[0];
    p.qs1 = a.q.stride[1];
    p.qs2 = a.q.stride[2];
    p.qs3 = a.q.stride[3];
    p.kc = a.k_cache;
    p.vc = a.v_cache;
    p.ksc = a.k_scale;
    p.vsc = a.v_scale;
    p.ptab = a.page_table;
    p.ctx = a.ctx_lens;
    p.T = a.T;
    p.H = a.H;
    p.Hk = a.Hk;
    p.G = a.H / a.Hk;
    p.R = a.T * p.G;
    p.Rpad = static_cast<int>(round_up(p.R, 16));
    p.page = a.page_size;
    p.max_pages = a.max_pages;
    p.num_pages = a.num_pages;
    p.window = a.window;
    p.nsplit = nsplit_for(a.T, a.window);
    p.logit_scale_log2 = a.softmax_scale / static_cast<float>(a.D) * kLog2e;
    p.part = static_cast<float*>(a.ws);
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.os0 = a.out_stride[0];
    p.os1 = a.out_stride[1];
    p.os2 = a.out_stride[2];
    p.os3 = a.out_stride[3];
    p.q_vec = (a.q.stride[3] == 1 && a.q.stride[0] % 8 == 0 && a.q.stride[1] % 8 == 0 &&
               a.q.stride[2] % 8 == 0 && reinterpret_cast<uintptr_t>(a.q.ptr) % 16 == 0)
                  ? 1
                  : 0;
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, DecSmem::kBytes);
    if (e != cudaSuccess) return e;
    decode_split_kernel<<<dim3(p.nsplit, a.B * a.Hk), kDecThreads, DecSmem::kBytes, s>>>(p);
    decode_combine_kernel<<<dim3(p.R, a.B * a.Hk), kD, 0, s>>>(p);
    return cudaGetLastError();
}

unsigned read_clear_decode_error() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_decode_err, sizeof v) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_decode_err, &zero, sizeof zero);
    return v;
}

}  // namespace sage
