// decode.cu -- paged FP8-KV decode with MTP query tokens, GQA and a sliding
// window ("[FlyDSL] [Misc] pa_decode: key the tile kernel on FlyDSL dtypes
// and drop the batch-first plan grid": window-family workload with per-token
// FP8 K/V scales, MTP4, GQA16, one KV head, page 128; Changes: Q/P quantised
// to the FP8 format of the cache (Q here), PV on bf16 operands because a
// per-token V scale cannot be factored out of the sum).
//
// Split-KV. decode_split_kernel: CTA (split, b * Hk + hk), 4 warps, handles
// up to 256 consecutive keys of the union of the T query tokens' windows for
// all R = T * (H / Hk) query rows of kv head hk (16 rows per warp):
//   1. Q rows: bf16 -> fp32 butterfly rotation -> e4m3 with scale
//      max|q_hat| / 448 (same fp32 operations as the quantisation kernels);
//   2. per 64-key chunk: K and V rows gathered through the page table with
//      cp.async (page ids are bounds-checked), V decoded exactly to bf16;
//      S = Q8 K8^T with e4m3 mma.sync (fp32 accumulate), scaled by
//      s_q * s_k * softmax_scale / D, masked to each row's own window;
//      online softmax in base 2; P' = p * s_v rounded to bf16; O += P' V
//      with bf16 mma.sync;
//   3. (m, l, O) of every row to the workspace.
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
constexpr int kSplit = 256;                  // keys per CTA
constexpr int kChunk = 64;                   // keys per inner step
constexpr int kMaxRows = 64;                 // T * (H / Hk)
constexpr int kKPitch = kD + 16;             // bytes per K row in smem
constexpr int kVPitch = kD + 8;              // bf16 elements per V row in smem
constexpr float kLog2e = 1.4426950408889634f;

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

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
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

__global__ void __launch_bounds__(128) decode_split_kernel(const DecParams p) {
    __shared__ __align__(16) uint8_t q8s[kMaxRows][kD];
    __shared__ float sq[kMaxRows];
    __shared__ __align__(16) uint8_t ks8[kChunk][kKPitch];
    __shared__ __align__(16) uint8_t vs8[kChunk][kD];
    __shared__ __align__(16) __nv_bfloat16 vbf[kChunk][kVPitch];
    __shared__ float kscl[kChunk], vscl[kChunk];
    __shared__ int tok_ok[kChunk];

    const int split = blockIdx.x, bhk = blockIdx.y;
    const int b = bhk / p.Hk, hk = bhk % p.Hk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tg = lane & 3;

    int ctx = p.ctx[b];
    const int cap = p.max_pages * p.page;
    if (ctx > cap || ctx < 0) {
        if (tid == 0 && split == 0) atomicCAS(&g_decode_err, 0u, kErrDecodeRange);
        ctx = max(0, min(ctx, cap));
    }
    const int lo = max(0, ctx - p.T - p.window + 1);
    const int k_begin = lo + split * kSplit;
    const int k_end = min(ctx, k_begin + kSplit);      // exclusive

    // ---- 1. query rows: rotate and quantise to e4m3 (one thread per row)
    if (tid < kMaxRows) {
        const int r = tid;
        if (r < p.R) {
            const int t = r / p.G, h = hk * p.G + r % p.G;
            const uint16_t* src = p.q + b * p.qs0 + t * p.qs1 + h * p.qs2;
            float x[kD];
#pragma unroll
            for (int d = 0; d < kD; ++d)
                x[d] = __uint_as_float(static_cast<uint32_t>(__ldg(src + d * p.qs3)) << 16);
#pragma unroll
            for (int lg = 0; lg < 7; ++lg) {
                const int hh = 1 << lg;
#pragma unroll
                for (int kk = 0; kk < kD / 2; ++kk) {
                    const int j = ((kk >> lg) << (lg + 1)) + (kk & (hh - 1));
                    const float a = x[j], c = x[j + hh];
                    x[j] = __fadd_rn(a, c);
                    x[j + hh] = __fsub_rn(a, c);
                }
            }
            float amax = 0.0f;
#pragma unroll
            for (int d = 0; d < kD; ++d) amax = fmaxf(amax, fabsf(x[d]));
            float s = 0.0f, rr = 0.0f;
            if (amax != 0.0f) {
                s = __fdiv_rn(amax, 448.0f);
                rr = __fdiv_rn(448.0f, amax);
            }
            sq[r] = s;
#pragma unroll
            for (int d = 0; d < kD; d += 4) {
                const uint32_t lo16 = e4m3x2_rn_satfinite(__fmul_rn(x[d], rr), __fmul_rn(x[d + 1], rr));
                const uint32_t hi16 = e4m3x2_rn_satfinite(__fmul_rn(x[d + 2], rr), __fmul_rn(x[d + 3], rr));
                *reinterpret_cast<uint32_t*>(&q8s[r][d]) = lo16 | (hi16 << 16);
            }
        } else {
            sq[r] = 0.0f;
#pragma unroll
            for (int d = 0; d < kD; d += 16) *reinterpret_cast<uint4*>(&q8s[r][d]) = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();

    // A fragments of this warp's 16 rows (4 k-steps of 32 channels), kept in registers
    const int row0 = warp * 16;
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
    const bool va = ra < p.R, vb = rb < p.R;
    const int pa = va ? ctx - p.T + ra / p.G : -1;      // query position of each row
    const int pb = vb ? ctx - p.T + rb / p.G : -1;
    const float ca = va ? sq[ra] * p.logit_scale_log2 : 0.0f;
    const float cb = vb ? sq[rb] * p.logit_scale_log2 : 0.0f;

    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;

    for (int c0 = k_begin; c0 < k_end; c0 += kChunk) {
        const int nk = min(kChunk, k_end - c0);
        __syncthreads();          // previous chunk's smem reads are done
        // ---- 2a. gather K and V rows (16 B pieces) through the page table
        for (int i = tid; i < kChunk * (kD / 16); i += 128) {
            const int kr = i / (kD / 16), piece = i % (kD / 16);
            const int j = c0 + kr;
            bool ok = kr < nk;
            int64_t tok = 0;
            if (ok) {
                const int pg = __ldg(&p.ptab[(int64_t)b * p.max_pages + j / p.page]);
                if (pg < 0 || pg >= p.num_pages) {
                    ok = false;
                    atomicCAS(&g_decode_err, 0u, kErrDecodeRange);
                } else {
                    tok = ((int64_t)pg * p.Hk + hk) * p.page + (j % p.page);
                }
            }
            cp_async16(&ks8[kr][piece * 16], p.kc + (ok ? tok * kD + piece * 16 : 0), ok);
            cp_async16(&vs8[kr][piece * 16], p.vc + (ok ? tok * kD + piece * 16 : 0), ok);
            if (piece == 0) {
                kscl[kr] = ok ? __ldg(&p.ksc[tok]) : 0.0f;
                vscl[kr] = ok ? __ldg(&p.vsc[tok]) : 0.0f;
                tok_ok[kr] = ok ? 1 : 0;
            }
        }
        cp_async_wait_all();
        __syncthreads();
        // V e4m3 -> bf16 (exact)
        for (int i = tid; i < kChunk * (kD / 4); i += 128) {
            const int kr = i / (kD / 4), c4 = (i % (kD / 4)) * 4;
            uint32_t lo2, hi2;
            e4m3x4_to_bf16x4(*reinterpret_cast<const uint32_t*>(&vs8[kr][c4]), lo2, hi2);
            *reinterpret_cast<uint2*>(&vbf[kr][c4]) = make_uint2(lo2, hi2);
        }
        __syncthreads();

        // ---- 2b. S = Q8 K8^T for 64 keys (8 n-tiles of 8 keys)
        float sacc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.0f;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&ks8[nt * 8 + g][kk * 32 + tg * 4]);
                const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&ks8[nt * 8 + g][kk * 32 + 16 + tg * 4]);
                mma_e4m3_16832(sacc[nt], qa[kk], b0, b1);
            }
        }
        // scale, mask to each row's window, base-2 logits
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kr = nt * 8 + tg * 2 + e;
                const int j = c0 + kr;
                const float ksv = kscl[kr];
                const bool okk = kr < nk && tok_ok[kr];
                const bool vis_a = okk && j <= pa && j > pa - p.window;
                const bool vis_b = okk && j <= pb && j > pb - p.window;
                sacc[nt][e] = vis_a ? sacc[nt][e] * ca * ksv : -INFINITY;
                sacc[nt][2 + e] = vis_b ? sacc[nt][2 + e] * cb * ksv : -INFINITY;
                mx_a = fmaxf(mx_a, sacc[nt][e]);
                mx_b = fmaxf(mx_b, sacc[nt][2 + e]);
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
                const int kr = nt * 8 + tg * 2 + e;
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
                ldmatrix_x4_trans(bfr, &vbf[krow][col]);
                mma_bf16_16816(o[2 * np], afr, bfr[0], bfr[1]);
                mma_bf16_16816(o[2 * np + 1], afr, bfr[2], bfr[3]);
            }
        }
    }

    // ---- 3. partial results of this split
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
    decode_split_kernel<<<dim3(p.nsplit, a.B * a.Hk), 128, 0, s>>>(p);
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
