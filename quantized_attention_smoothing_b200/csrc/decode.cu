// decode.cu -- paged FP8-KV decode with MTP query tokens, GQA and a sliding
// window ("[FlyDSL] [Misc] pa_decode: key the tile kernel on FlyDSL dtypes
// and drop the batch-first plan grid": window-family workload with per-token
// FP8 K/V scales, MTP4, GQA16, one KV head, page 128; Changes: Q/P quantised
// to the FP8 format of the cache (Q here), PV on bf16 operands because a
// per-token V scale cannot be factored out of the sum).
//
// Two kernels. The keys of sequence b (the union of its T query tokens'
// windows, [lo, ctx)) are cut into 128-key tiles aligned to absolute key
// positions, so a tile is one page (page 128) or 128 / page whole pages.
// The tiles of (b, kv head hk) are shared out among up to 16 CTAs of
// decode_kernel (the count is picked at launch so that the grid runs in one
// wave, one CTA per SM); CTA = 16 warps:
//   warps 0-7  softmax, two groups: warps 0-3 take the even tiles, warps 4-7
//              the odd ones, each group with its own running max and sum
//              and its own O accumulator; warp w of a group owns A rows
//              16 (w & 3) .. + 15 of the QK operand (R = T * H/Hk query
//              rows, row r = t * G + g, padded to 64; with R <= 32 the rows
//              repeated NREP = 2 or 4 times, and the warp takes 128 / NREP
//              of the key columns) -- M = 64 MMAs keep those rows in TMEM
//              lanes 32 (w & 3) .. + 15;
//   warps 8-11 V converters: e4m3 V tile -> exact bf16 (integer bit
//              placement and one bf16 multiply), in the key order of the P
//              operand (an MXFP4 cache: K and V tiles -> exact bf16);
//   warp 12    K/V producer: page-table lookups, one TMA box per page for K
//              and for V;
//   warp 13    TMEM owner and MMA issuer;
//   warp 14    scale producer: per-token scales by cp.async and the tile's
//              bad-page mask, on a ring of their own (warp 15 only completes
//              the producers' warpgroup).
// Per tile: S = Q8 K8^T (e4m3 tcgen05 MMAs, M=64 N=128, fp32 in TMEM,
// double-buffered by tile parity) -> base-2 logits (S * k_scale_j) * s_q *
// softmax_scale / D, masked to each row's own window -> the group's running
// max m -> p = 2^(x - m) -> P' = bf16(p * v_scale_j) -> O[i & 1] += P' V
// (bf16 tcgen05 MMAs, M=64 N=128, fp32 in TMEM). Before PV(i), the rows of
// O[i & 1] whose group max rose since tile i - 2 are rescaled by 2^(m_old -
// m); after the last tile the two groups' (m, l, O) are combined. The query
// rows are rotated and quantised to e4m3 in the prologue (fp32 butterfly,
// four threads per row, scale max|q_hat| / 448, the operations of the
// quantisation kernels). A CTA that holds every tile of (b, hk) writes bf16
// through the caller's strides; otherwise every CTA writes its (m, l, O) to
// the workspace and decode_merge_kernel, launched after it on the stream,
// combines the splits (log-sum-exp) and writes bf16.
//
// The MXFP4 cache (same page, Changes: a uint8 cache is MXFP4, E4M3 for the
// query): E2M1 codes with one e8m0 exponent per 32 elements, converted to
// exact bf16 in shared memory (K into one buffer that each QK frees, V as
// above); QK is then a bf16 MMA on the query codes widened to bf16, and the
// key and value scales are 1.
//
// Every mbarrier wait is bounded; on timeout the CTA records an error word,
// raises its abort flag, drains its own copies and MMAs and still reaches
// its CTA barriers.
#include <algorithm>
#include <cfloat>
#include <climits>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {
namespace {

__device__ unsigned g_decode_err;
constexpr unsigned kErrDecodeRange = kErrRangeCode;   // ctx or page id out of range (clamped / masked)

constexpr int kKeys = 128;                   // keys per tile
constexpr int kRows = 64;                    // query rows per CTA (M of every MMA)
constexpr int kStages = 3;                   // K / V ring
constexpr int kScStages = 8;                 // per-token scale ring (freed by the softmax alone)
constexpr int kMaxSplit = 16;                // CTAs per (sequence, kv head)
constexpr int kSoftWarps = 8;                // warps 0..7
constexpr int kConvWarp0 = 8;                // warps 8..11
constexpr int kTmaWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kScaleWarp = 14;
constexpr int kIdleWarp = 15;                // initialises the barriers, then only completes a warpgroup
constexpr int kThreads = 512;
// registers per thread of each warpgroup (setmaxnreg; 256 x 168 + 128 x 96 +
// 128 x 80 <= 512 x 128, the launch's registers; this split compiles without
// spills at both head sizes). Only the softmax warps ever grow their share,
// after the others have shrunk theirs, and no warp grows it again later: a
// warp that did could take registers another one waits for.
constexpr int kRegsSoft = 168, kRegsConv = 96, kRegsProd = 80;
static_assert(2 * 128 * kRegsSoft + 128 * kRegsConv + 128 * kRegsProd <= 512 * 128, "register split");
// the MXFP4 cache's kernels: the split that compiles without spills for
// each row-repeat count (the converters do K and V there)
template <bool MX, int NREP> struct RegSplit {
    static constexpr int soft = kRegsSoft, conv = kRegsConv, prod = kRegsProd;
};
template <int NREP> struct RegSplit<true, NREP> {
    static constexpr int soft = 168, conv = NREP == 2 ? 80 : 96, prod = NREP == 2 ? 96 : 80;
    static_assert(2 * 128 * soft + 128 * conv + 128 * prod <= 512 * 128, "register split");
};
constexpr float kLog2e = 1.4426950408889634f;
// A scale slot: k_scale then v_scale of the tile's keys, each by key parity
// (index (key & 1) * kScPar + key / 2); the 4-float pad puts the two parities'
// 16-byte reads in different banks
constexpr int kScPar = kKeys / 2 + 4, kScHalf = 2 * kScPar, kScSlot = 2 * kScHalf;

// Head size D (64 or 128): an e4m3 row of Q, K or V is D bytes, stored
// with the swizzle of that span (128B or 64B); a bf16 V row is 2 D bytes,
// one or two 64-channel 128B-swizzled atoms.
// The 16-byte chunk c of row r of a D-byte swizzled e4m3 row tile.
template <int D>
__device__ __forceinline__ int e4m3_chunk(int c, int r) {
    return D == 128 ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3));
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// 16 registers from 16 TMEM lanes (shape 16x64b, x16): the mapping of
// tmem_ld16x64 over 32 columns. Valid after tmem_wait_ld16(r).
__device__ __forceinline__ void tmem_ld16x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x64b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                   "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
}

// N registers of 16 TMEM lanes and 2 N columns (shape 16x64b), loaded and
// waited for: N = 32 or 16.
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld16x32(taddr, r);
    tmem_wait_ld(r);
}
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, uint32_t (&r)[16]) {
    tmem_ld16x16(taddr, r);
    tmem_wait_ld16(r);
}

constexpr int al1024(int x) { return (x + 1023) & ~1023; }

// N registers of 16 TMEM lanes and 2 N columns (shape 16x64b), loaded and
// waited for: N = 64, 32 or 16.
__device__ __forceinline__ void tmem_ld16_cols(uint32_t taddr, uint32_t (&r)[64]) {
    tmem_ld16x64(taddr, r);
    tmem_wait_ld64(r);
}
__device__ __forceinline__ void tmem_ld16_cols(uint32_t taddr, uint32_t (&r)[32]) { tmem_ld16_wait(taddr, r); }
__device__ __forceinline__ void tmem_ld16_cols(uint32_t taddr, uint32_t (&r)[16]) { tmem_ld16_wait(taddr, r); }

// dynamic shared memory (offsets from a 1024-byte aligned base). MX: the
// cache holds E2M1 codes with e8m0 block scales (head size 128), the query
// rows are bf16 and K is converted to bf16 before QK.
template <int D, bool MX = false>
struct SmL {
    static constexpr int kOcPitch = D + 4;                         // fp32 row pitch of the merge area
    static constexpr int kQ = 0;                                   // [64][D] e4m3, MX: bf16 [2 atoms][64][128 B]
    static constexpr int kKStage = MX ? kKeys * D / 2 : kKeys * D; // codes of one tile: [128][D] e4m3 | [128][D / 2] E2M1
    static constexpr int kK = kQ + (MX ? 2 : 1) * kRows * D;       // [stage] K codes
    static constexpr int kV = kK + kStages * kKStage;              // [stage] V codes (V^T: [D][128])
    static constexpr int kSfStage = MX ? kKeys * D / 32 : 0;       // MX: e8m0 block scales of one tile [128][D / 32]
    static constexpr int kKsf = kV + kStages * kKStage;
    static constexpr int kVsf = kKsf + kStages * kSfStage;
    static constexpr int kKbBuf = MX ? kKeys * 2 * D : 0;          // MX: bf16 K, D / 64 channel atoms [128][128 B]
    static constexpr int kKb = MX ? al1024(kVsf + kStages * kSfStage) : kVsf;
    static constexpr int kPBuf = 2 * kRows * 128;                  // two 64-key atoms [64][128 B] bf16
    static constexpr int kP = kKb + kKbBuf;                        // [2 bufs] P' (A of PV)
    static constexpr int kVbBuf = kKeys * 2 * D;                   // D / 64 channel atoms [128][128 B] bf16
    static constexpr int kVb = kP + 2 * kPBuf;                     // [2 bufs] bf16 V (B of PV)
    static constexpr int kScale = kVb + 2 * kVbBuf;                // [slot] ks | vs fp32, padded
    static constexpr int kSq = kScale + kScStages * kScSlot * 4;   // [64] fp32 query scales
    static constexpr int kMeta = kSq + kRows * 4;                  // [slot] int: pages with a bad id
    static constexpr int kGrp = kMeta + kScStages * 4;             // [m | l][tile parity][64] fp32
    static constexpr int kBar = kGrp + 2 * 2 * kRows * 4;
    // barriers
    static constexpr int kKvFull = 0, kKvEmpty = kKvFull + kStages, kSFull = kKvEmpty + kStages,
                         kPReady = kSFull + 2, kPvDone = kPReady + 2, kFinal = kPvDone + 2,
                         kQReady = kFinal + 1, kScFull = kQReady + 1, kScEmpty = kScFull + kScStages,
                         kKbReady = kScEmpty + kScStages, kKbFree = kKbReady + 1,
                         kNumBars = kKbFree + 1;
    static constexpr int kMisc = kBar + kNumBars * 8;              // TMEM base, abort flag
    static constexpr int kBytes = kMisc + 16;
    // merge area, over the K (and, MX, V) code stages (free once the last
    // tile is consumed)
    static constexpr int kOc = kK;                                 // [64][kOcPitch] fp32
    static constexpr int kStat = kOc + kRows * kOcPitch * 4;       // [64] (m, l)
    static_assert(kOcPitch % 4 == 0, "merge rows are 16-byte aligned");
    static_assert(kStat + kRows * 8 <= (MX ? kKsf : kV), "merge area fits in the code stages");
    static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kP % 1024 == 0 && kVb % 1024 == 0 &&
                      kKb % 1024 == 0 && kKsf % 16 == 0,
                  "swizzled tiles are 1024-byte aligned");
    static_assert(kBytes + 1024 <= 227 * 1024, "shared memory");
    static_assert(D == 64 || D == 128, "head size");
    static_assert(!MX || D == 128, "the MXFP4 cache is read at head size 128");
};

struct DecParams {
    const uint16_t* q;
    int64_t qs0, qs1, qs2, qs3;              // q strides [B, T, H, D] (elements)
    const float* ksc;
    const float* vsc;
    const int32_t* ptab;
    const int32_t* ctx;
    int T, H, Hk, G, R, page, lg_page, max_pages, num_pages, window, nsplit;
    int q_vec;                               // q rows contiguous and 16-byte aligned
    float logit_scale_log2;                  // softmax_scale / D * log2(e)
    __nv_bfloat16* out;
    int64_t os0, os1, os2, os3;
    uint8_t* q8_out;                         // optional: e4m3 query codes [B, T, H, D]
    float* qs_out;                           // optional: query scales [B, T, H]
    int per_tensor;                          // ksc / vsc hold one scale each
    int v_trans;                             // V cache [num_pages, Hk, D, page] (page 128)
    int o_vec;                               // out rows: 4 channels as one 8-byte store
    const uint8_t* ksf8;                     // MX: e8m0 block scales [num_pages, Hk, page, D / 32]
    const uint8_t* vsf8;
    float2* ws_stat;                         // nsplit > 1: partial (m, l) [B Hk][nsplit][64]
    float* ws_o;                             //   and partial O [B Hk][nsplit][64][128] fp32
};

// The A operand (P') of the PV MMA holds a row's 128 keys in this order:
// position 16i + 8c + m <-> key 16i + c + 2m (c = 0, 1; m = 0..7), which
// is what a softmax thread holds (its columns have one parity c), so it
// writes 16 contiguous bytes per 16 keys. V rows are stored in the same
// order.
__device__ __forceinline__ int pv_position(int key) {
    return (key & ~15) + 8 * (key & 1) + ((key & 15) >> 1);
}

// e4m3 codes -> bf16 with exactly the same values, integer operations only.
// A code's 7 magnitude bits placed at bf16 bits 4..10 and its sign at bit 15
// read as a bf16 of value x * 2^-120 (exponent field e of a normal code kept,
// a subnormal code a bf16 subnormal), and the bf16 product by 2^120 is exact.
// `sel` picks the two code bytes of `w` (0x1404: bytes 0, 1; 0x3424: 2, 3).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w, uint32_t sel) {
    const uint32_t t = __byte_perm(w, 0u, sel);          // code bytes at bits 8..15 and 24..31
    const uint32_t bits = ((t >> 4) & 0x07F007F0u) | (t & 0x80008000u);
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(bits), "r"(0x7B807B80u));   // 2^120
    return r;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// The e4m3 codes byte m of `a` and byte m of `b` as one bf16 pair (low half
// from `a`), exactly, as in e4m3x2_to_bf16x2; m = 0..3.
template <int m>
__device__ __forceinline__ uint32_t e4m3_pick_to_bf16x2(uint32_t a, uint32_t b) {
    const uint32_t t = __byte_perm(a, b, (m << 4) | ((4 + m) << 12));   // bytes 1 and 3; 0, 2 unused
    return bf16x2_mul(((t >> 4) & 0x07F007F0u) | (t & 0x80008000u), 0x7B807B80u);
}

// Eight E2M1 codes (OCP MX: sign, two exponent bits, one mantissa bit),
// nibble i of `w` (bits 4i .. 4i + 3) holding element i, as four bf16 pairs:
// pair m = (element m, element m + 4), each times the bf16 pair `c2`.
// A code's three magnitude bits placed at bf16 bits 6..8 and its sign at bit
// 15 read as a bf16 of value x * 2^-126 (exponent field = the code's, a
// zero-exponent code a bf16 subnormal), so c2 = 2^(E - 1) gives x * 2^(E -
// 127) in one exact product while that is a bf16 value.
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t w, uint32_t c2, uint32_t* o) {
    const uint32_t a0 = w << 6, a1 = w << 2, a2 = w >> 2, a3 = w >> 6;
    const uint32_t s0 = w << 12, s1 = w << 8, s2 = w << 4, s3 = w;
    o[0] = bf16x2_mul((a0 & 0x01C001C0u) | (s0 & 0x80008000u), c2);
    o[1] = bf16x2_mul((a1 & 0x01C001C0u) | (s1 & 0x80008000u), c2);
    o[2] = bf16x2_mul((a2 & 0x01C001C0u) | (s2 & 0x80008000u), c2);
    o[3] = bf16x2_mul((a3 & 0x01C001C0u) | (s3 & 0x80008000u), c2);
}

// One MX block (32 E2M1 codes, 16 bytes: elements 8g .. 8g + 7 in word g)
// times 2^(E - 127), E its e8m0 scale code, as 16 bf16 pairs: pair 4g + m =
// (element 8g + m, element 8g + m + 4). E is read as min(E, 252), the largest
// exponent whose values (up to 6 * 2^125) are finite in bf16, so that cache
// bytes the window masks (slots past ctx) cannot turn a zero weight into a
// NaN; a larger E (and E = 255, NaN) lies outside the contract.
__device__ __forceinline__ void e2m1_block_to_bf16(uint4 u, uint32_t E, uint32_t (&o)[16]) {
    E = min(E, 252u);
    const uint32_t lo = E <= 128u ? E + 126u : 253u;                  // 2^(E - 1), or 2^126 then 2^(E - 127)
    const uint32_t c2 = (lo << 7) | (lo << 23);
    e2m1x8_to_bf16(u.x, c2, o);
    e2m1x8_to_bf16(u.y, c2, o + 4);
    e2m1x8_to_bf16(u.z, c2, o + 8);
    e2m1x8_to_bf16(u.w, c2, o + 12);
    if (E > 128u) {
        const uint32_t c3 = (E << 7) | (E << 23);
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = bf16x2_mul(o[k], c3);
    }
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// Barrier `id` (1..15) of `count` threads (whole warps).
__device__ __forceinline__ void named_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// CTA-wide barrier in its non-aligned form: the threads may reach it from
// different code (each thread arrives exactly once).
__device__ __forceinline__ void bar_sync_all(int count) {
    asm volatile("bar.sync 0, %0;" ::"r"(count) : "memory");
}

// Output row rr of (b, hk), channels d4 .. d4 + 3: o * inv as bf16 through
// the caller's strides.
__device__ __forceinline__ void store_out4(const DecParams& p, int b, int hk, int rr, int d4, float4 o,
                                           float inv) {
    const int t = rr / p.G, h = hk * p.G + rr % p.G;
    __nv_bfloat16* dst = p.out + b * p.os0 + t * p.os1 + h * p.os2 + (int64_t)d4 * p.os3;
    const __nv_bfloat162 y01 = __floats2bfloat162_rn(o.x * inv, o.y * inv);
    const __nv_bfloat162 y23 = __floats2bfloat162_rn(o.z * inv, o.w * inv);
    if (p.o_vec) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<const uint32_t*>(&y01),
                                                    *reinterpret_cast<const uint32_t*>(&y23));
    } else {
        dst[0] = y01.x;
        dst[p.os3] = y01.y;
        dst[2 * p.os3] = y23.x;
        dst[3 * p.os3] = y23.y;
    }
}

// NREP (1, 2, 4): the R <= 64 / NREP query rows are repeated NREP times in
// the 64 rows of the QK A operand, row r holding query row r % (64 / NREP),
// and warp qw of a softmax group takes the 128 / NREP key columns of its
// 16 rows that begin at (qw / (4 / NREP)) * 128 / NREP: with few query rows
// (one query token: R = H / Hk) every softmax warp then holds a share of the
// logits instead of one warp holding them all. Each A row keeps its own
// running max, sum and O rows; the NREP rows of a query row are combined
// (log-sum-exp) with the two groups' when the CTA's result is written.
template <int D, bool MX, int NREP>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecParams p) {
    using Sm = SmL<D, MX>;
    static_assert(NREP == 1 || NREP == 2 || NREP == 4, "row repeats");
    constexpr int kPeriod = kRows / NREP;         // query rows per repeat of the A operand
    constexpr int kNC = 64 / NREP;                // S registers per softmax thread (2 kNC columns a row)
    constexpr int kD = D;
    constexpr int kOcPitch = Sm::kOcPitch;
    constexpr int kQe = D / 4;                    // query elements per rotating thread (4 per row)
    constexpr int kQv = D / 32;                   // their 16-byte loads
    constexpr int kLgQe = D == 128 ? 5 : 4;       // butterfly stages inside a thread
    constexpr int kOe = D / 4;                    // output registers per epilogue thread (D / 2 columns)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Sm::kBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Sm::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Sm::kMisc + 4);
    float* sq = reinterpret_cast<float*>(sm + Sm::kSq);
    int* meta = reinterpret_cast<int*>(sm + Sm::kMeta);
    float* scl = reinterpret_cast<float*>(sm + Sm::kScale);

    const int split = blockIdx.x;
    const int bhk = blockIdx.y;
    const int b = bhk / p.Hk, hk = bhk % p.Hk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // setup that reads no global memory (barriers, TMEM, the tensor maps of
    // the parameter space) overlaps the preceding kernel in the stream when
    // this grid is launched as its programmatic dependent; everything after
    // griddepcontrol.wait sees that kernel's writes
    // softmax warps per group that hold query rows (the others, whose 16
    // rows are all padding, take no part in the tile loop)
    const int n_act = NREP > 1 ? 4 : min(4, (p.R + 15) >> 4);
    if (warp == kIdleWarp) {
        for (int i = lane; i < Sm::kNumBars; i += 32) {
            uint32_t cnt = 1;                                       // expect_tx; commits
            if (i >= Sm::kKvEmpty && i < Sm::kKvEmpty + kStages) cnt = MX ? 4 : 1 + 4;  // (QK commit +) converters
            if (i >= Sm::kPReady && i < Sm::kPReady + 2) cnt = n_act + 4;         // softmax group + converters
            if (i == Sm::kQReady) cnt = kSoftWarps;
            if (i >= Sm::kScFull && i < Sm::kScFull + kScStages) cnt = 1 + 32;    // bad-page mask + scale copies
            if (i >= Sm::kScEmpty && i < Sm::kScEmpty + kScStages) cnt = n_act;   // softmax group
            if (i == Sm::kKbReady) cnt = 4;                                       // converters (MX)
            mbar_init(&bars[i], cnt);
        }
        if (lane == 0) *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == kTmaWarp && lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    pdl_wait();
    pdl_launch_dependents();

    int ctx = p.ctx[b];
    const int cap = p.max_pages * p.page;
    if (ctx > cap || ctx < 0) {
        if (tid == 0 && split == 0) atomicCAS(&g_decode_err, 0u, kErrDecodeRange);
        ctx = max(0, min(ctx, cap));
    }
    // keys [lo, ctx) as 128-key tiles [t0, t1) at absolute positions; this
    // CTA's share is [tb, tb + nt)
    const int lo = max(0, ctx - p.T - p.window + 1);
    const int t0 = lo / kKeys, t1 = (ctx + kKeys - 1) / kKeys;
    const int n_all = max(0, t1 - t0);
    const int tb = t0 + (split * n_all) / p.nsplit;
    const int nt = t0 + ((split + 1) * n_all) / p.nsplit - tb;

    // the producer's first page-table entries, requested before the barrier
    const int ppt = kKeys / p.page;                  // pages per tile (divides 32)
    int pg_first = 0;
    if (warp == kTmaWarp || warp == kScaleWarp) {
        const int lp = tb * ppt + lane;
        if (lp < (tb + nt) * ppt && lp * p.page < ctx && lp * p.page + p.page > lo)
            pg_first = __ldg(&p.ptab[(int64_t)b * p.max_pages + lp]);
    }
    // the softmax warps' query row quarters (contiguous rows), also in flight
    // across the barrier
    uint4 qv[kQv] = {};
    if (warp < kSoftWarps && p.q_vec && ((tid >> 2) % kPeriod) < p.R) {
        const int r = (tid >> 2) % kPeriod;
        const uint4* src = reinterpret_cast<const uint4*>(p.q + b * p.qs0 + (r / p.G) * p.qs1 +
                                                          (hk * p.G + r % p.G) * p.qs2) + kQv * (tid & 3);
#pragma unroll
        for (int c = 0; c < kQv; ++c) qv[c] = __ldg(src + c);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM columns: S double buffer [0, 256); O of even tiles [256, 384), of
    // odd tiles [384, 512)
    constexpr uint32_t kOCol = 256;


    if (warp >= kTmaWarp) {
      reg_dealloc<RegSplit<MX, NREP>::prod>();
      if (warp == kTmaWarp || warp == kScaleWarp) {
        // ------------------------------------------------------------ producers
        // Both warps look up the physical pages of the CTA's logical pages
        // tb * ppt + 32 c + lane, 32 at a time (lane j of chunk c holds page
        // 32 c + j); pages holding no key of [lo, ctx) are not looked up
        // (page 0 stands in; their keys are masked). Warp 12 loads K and V
        // by TMA, the lanes of a tile's pages each issuing their own boxes;
        // warp 14 loads the per-token scales and the tile's bad-page mask.
        const bool kv = warp == kTmaWarp;
        // MX: the block scales are applied in the conversion, so every key's
        // k_scale and v_scale are 1
        const bool per_tensor = MX || p.per_tensor;
        const float ks_tensor = MX ? 1.0f : (!kv && per_tensor) ? __ldg(p.ksc) : 0.0f;
        const float vs_tensor = MX ? 1.0f : (!kv && per_tensor) ? __ldg(p.vsc) : 0.0f;
        int chunk = -1, phys_l = 0;
        bool bad_l = false;
        int issued = 0;
        for (int i = 0; i < nt; ++i) {
            const int s = i % kStages, c = i % kScStages;
            const bool free_slot =
                kv ? mbar_wait(&bars[Sm::kKvEmpty + s], ((i / kStages) & 1) ^ 1, abort_flag, &g_decode_err, 1)
                   : mbar_wait(&bars[Sm::kScEmpty + c], ((i / kScStages) & 1) ^ 1, abort_flag, &g_decode_err, 7);
            if (!warp_all(free_slot)) break;
            if ((i * ppt) / 32 != chunk) {
                chunk = (i * ppt) / 32;
                const int lp = tb * ppt + 32 * chunk + lane;
                const int k0 = lp * p.page;
                phys_l = 0;
                bad_l = false;
                if (lp < (tb + nt) * ppt && k0 < ctx && k0 + p.page > lo) {
                    const int pg = chunk == 0 ? pg_first : __ldg(&p.ptab[(int64_t)b * p.max_pages + lp]);
                    if (pg < 0 || pg >= p.num_pages) {
                        bad_l = true;
                        if (kv) atomicCAS(&g_decode_err, 0u, kErrDecodeRange);
                    } else {
                        phys_l = pg;
                    }
                }
            }
            const int slot0 = (i * ppt) % 32;             // this tile's pages: lanes slot0 .. slot0 + ppt - 1
            const bool mine = lane >= slot0 && lane < slot0 + ppt;
            if (kv) {
                if (lane == slot0)
                    mbar_arrive_expect_tx(&bars[Sm::kKvFull + s], 2 * (Sm::kKStage + Sm::kSfStage));
                __syncwarp();
                if (mine) {
                    const int z = phys_l * p.Hk + hk;
                    const int q = lane - slot0;
                    constexpr int kRowB = Sm::kKStage / kKeys;      // code bytes per key
                    tma_load_3d(sm + Sm::kK + s * Sm::kKStage + q * p.page * kRowB, &tmK, &bars[Sm::kKvFull + s], 0, 0, z);
                    tma_load_3d(sm + Sm::kV + s * Sm::kKStage + q * p.page * kRowB, &tmV, &bars[Sm::kKvFull + s], 0, 0, z);
                    if constexpr (MX) {
                        // the page's block scales, contiguous [page][D / 32]
                        constexpr int kSfB = kD / 32;
                        const int64_t off = (int64_t)z * p.page * kSfB;
                        bulk_load(sm + Sm::kKsf + s * Sm::kSfStage + q * p.page * kSfB, p.ksf8 + off,
                                  p.page * kSfB, &bars[Sm::kKvFull + s]);
                        bulk_load(sm + Sm::kVsf + s * Sm::kSfStage + q * p.page * kSfB, p.vsf8 + off,
                                  p.page * kSfB, &bars[Sm::kKvFull + s]);
                    }
                }
            } else {
                const unsigned badm = __ballot_sync(0xffffffffu, mine && bad_l) >> slot0;
                if (lane == 0) {
                    meta[c] = static_cast<int>(badm);
                    mbar_arrive(&bars[Sm::kScFull + c]);
                }
                // per-token scales of keys 4 lane .. 4 lane + 3, stored by key
                // parity for the softmax threads; with per-tensor scales the
                // one K and one V scale in every slot
                float* dst = scl + c * kScSlot;
                if (per_tensor) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = 4 * lane + e, at = (key & 1) * kScPar + (key >> 1);
                        dst[at] = ks_tensor;
                        dst[kScHalf + at] = vs_tensor;
                    }
                    mbar_arrive(&bars[Sm::kScFull + c]);
                } else {
                    const int kq = 4 * lane;
                    const int pq = __shfl_sync(0xffffffffu, phys_l, slot0 + kq / p.page);
                    const int64_t src = ((int64_t)pq * p.Hk + hk) * p.page + (kq % p.page);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = kq + e, at = (key & 1) * kScPar + (key >> 1);
                        cp_async_4(dst + at, p.ksc + src + e);
                        cp_async_4(dst + kScHalf + at, p.vsc + src + e);
                    }
                    cp_async_mbar_arrive(&bars[Sm::kScFull + c]);
                }
            }
            issued = i + 1;
        }
        // no copy of this CTA may land after it exits
        if (kv) {
            for (int i = max(0, issued - kStages); i < issued; ++i)
                mbar_wait_drain(&bars[Sm::kKvFull + i % kStages], (i / kStages) & 1);
        } else {
            for (int i = max(0, issued - kScStages); i < issued; ++i)
                mbar_wait_drain(&bars[Sm::kScFull + i % kScStages], (i / kScStages) & 1);
        }
      } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && nt > 0) {
            constexpr uint32_t kIdescQK = umma_idesc(1, MX ? 1 : 0, kRows, kKeys);     // e4m3 | bf16 -> f32
            constexpr uint32_t kIdescPV = umma_idesc(1, 1, kRows, kD) | (1u << 16);    // bf16, B MN-major
            constexpr uint32_t kIdescPVT = umma_idesc(1, 1, kRows, kD);                // bf16, B K-major
            const uint64_t qdesc = umma_desc_kmajor(smem_u32(sm + Sm::kQ), MX ? 128 : kD);
            // descriptors of the P' and V buffers, built once: a step of the
            // MMA loops only adds a constant to the start-address field
            // (V MN-major: two 64-channel swizzle atoms [128 keys][128 B], the
            // second one kKeys * 128 bytes on, the leading byte offset; V^T
            // converted K-major: 64-key atoms of [128 channels][128 B])
            const uint64_t vlbo = (p.v_trans || kD == 64) ? 0ull
                                                          : (static_cast<uint64_t>((kKeys * 128) >> 4) << 16) - (1ull << 16);
            const uint64_t pdesc0 = umma_desc_kmajor(smem_u32(sm + Sm::kP), 128);
            const uint64_t pdesc1 = umma_desc_kmajor(smem_u32(sm + Sm::kP + Sm::kPBuf), 128);
            const uint64_t vdesc0 = umma_desc_kmajor(smem_u32(sm + Sm::kVb), 128) + vlbo;
            const uint64_t vdesc1 = umma_desc_kmajor(smem_u32(sm + Sm::kVb + Sm::kVbBuf), 128) + vlbo;
            // S(i) = Q8 K8(i)^T into S buffer i & 1 (MX: bf16 Q and the
            // converters' bf16 K(i), two 64-channel atoms each, 16 channels a
            // step; the converters reuse the K buffer once this QK is done)
            auto issue_qk = [&](int i) -> bool {
                const int s = i % kStages;
                if constexpr (MX) {
                    if (!mbar_wait(&bars[Sm::kKbReady], i & 1, abort_flag, &g_decode_err, 2)) return false;
                    tc_fence_after();
                    const uint64_t kdesc = umma_desc_kmajor(smem_u32(sm + Sm::kKb), 128);
#pragma unroll
                    for (int st = 0; st < kD / 16; ++st)
                        mma_bf16_ss(tmem + 128 * (i & 1), qdesc + (st >> 2) * ((kRows * 128) >> 4) + 2 * (st & 3),
                                    kdesc + (st >> 2) * ((kKeys * 128) >> 4) + 2 * (st & 3), kIdescQK,
                                    st > 0 ? 1u : 0u);
                    mma_commit(&bars[Sm::kSFull + (i & 1)]);
                    mma_commit(&bars[Sm::kKbFree]);
                } else {
                    if (!mbar_wait(&bars[Sm::kKvFull + s], (i / kStages) & 1, abort_flag, &g_decode_err, 2))
                        return false;
                    tc_fence_after();
                    const uint64_t kdesc = umma_desc_kmajor(smem_u32(sm + Sm::kK + s * Sm::kKStage), kD);
#pragma unroll
                    for (int kk = 0; kk < kD / 32; ++kk)
                        mma_f8_ss(tmem + 128 * (i & 1), qdesc + 2 * kk, kdesc + 2 * kk, kIdescQK, kk > 0 ? 1u : 0u);
                    mma_commit(&bars[Sm::kSFull + (i & 1)]);
                    mma_commit(&bars[Sm::kKvEmpty + s]);
                }
                return true;
            };
            // order: QK(0), QK(1), then for j = 0, 1, ...: once P'(j) is
            // there, QK(j + 2) and PV(j). S(j + 2) overwrites S(j), which the
            // group read before it published P'(j); the group waits for PV(j)
            // itself before it reuses its P' buffer and O. (Measured slower:
            // issuing QK(j + 2) as soon as the group has read S(j); polling
            // for whichever of QK and PV can go next; the MX softmax groups
            // converting K of their own tiles.)
            auto k_there = [&](int i) -> bool {
                return MX ? mbar_test_wait(smem_u32(&bars[Sm::kKbReady]), i & 1)
                          : mbar_test_wait(smem_u32(&bars[Sm::kKvFull + i % kStages]), (i / kStages) & 1);
            };
            bool ok = mbar_wait(&bars[Sm::kQReady], 0, abort_flag, &g_decode_err, 12);
            if (ok) ok = issue_qk(0);
            if (ok && nt > 1) ok = issue_qk(1);
            for (int j = 0; ok && j < nt; ++j) {
                bool qk_next = false;
                ok = mbar_wait(&bars[Sm::kPReady + (j & 1)], (j >> 1) & 1, abort_flag, &g_decode_err, 4);
                if (!ok) break;
                // (FP8: PV first, measured faster -- the converters wait for it
                // before they reuse its V buffer; MX: QK first, which frees the
                // one bf16 K buffer the converters wait for)
                if (MX && j + 2 < nt && k_there(j + 2)) {
                    ok = issue_qk(j + 2);
                    qk_next = true;
                }
                // O[j & 1] += P'(j) V(j): 8 steps of 16 keys, all 128 channels
                // (P' atoms of 64 keys kRows * 128 bytes apart, 32 bytes per
                // 16 keys inside one; V: 2048 bytes per 16 keys, or V^T atoms
                // kD * 128 bytes apart and 32 bytes per 16 keys)
                tc_fence_after();
                const uint64_t pd = (j & 1) ? pdesc1 : pdesc0, vd = (j & 1) ? vdesc1 : vdesc0;
                const uint32_t odst = tmem + kOCol + kD * (j & 1);
                if (!p.v_trans) {
#pragma unroll
                    for (int st = 0; st < kKeys / 16; ++st)
                        mma_bf16_ss(odst, pd + (st >> 2) * ((kRows * 128) >> 4) + 2 * (st & 3), vd + 128 * st,
                                    kIdescPV, (j > 1 || st > 0) ? 1u : 0u);
                } else {
#pragma unroll
                    for (int st = 0; st < kKeys / 16; ++st)
                        mma_bf16_ss(odst, pd + (st >> 2) * ((kRows * 128) >> 4) + 2 * (st & 3),
                                    vd + (st >> 2) * ((kD * 128) >> 4) + 2 * (st & 3), kIdescPVT,
                                    (j > 1 || st > 0) ? 1u : 0u);
                }
                mma_commit(&bars[Sm::kPvDone + (j & 1)]);
                if (ok && j + 2 < nt && !qk_next) ok = issue_qk(j + 2);
            }
            // drain every MMA this thread issued before TMEM is released
            mma_commit(&bars[Sm::kFinal]);
            mbar_wait_drain(&bars[Sm::kFinal], 0);
        }
      }
        tc_fence_before();
        bar_sync_all(kThreads);
        if (warp == kMmaWarp) {                     // TMEM is read by nobody any more
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, 512);
        }
    } else if (warp < kSoftWarps) {
      reg_alloc<RegSplit<MX, NREP>::soft>();
        // ------------------------------------------------------------ softmax
        // ---- query rows: rotate and quantise to e4m3, four threads per row
        // (thread qq holds elements [32 qq, 32 qq + 32)), written as the
        // K-major 128B-swizzled A operand of QK. Every thread of warps 0-7
        // runs the whole sequence, shuffles included; rows past R load zeros,
        // which gives them zero codes and a zero scale.
        {
            const int r = tid >> 2, qq = tid & 3;          // A row r holds query row rq
            const int rq = r % kPeriod;
            const bool rv = rq < p.R;
            const int t = rv ? rq / p.G : 0, h = rv ? hk * p.G + rq % p.G : 0;
            const uint16_t* src = p.q + b * p.qs0 + t * p.qs1 + h * p.qs2 + (int64_t)(qq * kQe) * p.qs3;
            float x[kQe];
            if (p.q_vec) {
#pragma unroll
                for (int c = 0; c < kQv; ++c) {
                    const uint32_t wd[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};   // zeros past R
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        x[8 * c + 2 * e] = __uint_as_float(wd[e] << 16);
                        x[8 * c + 2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u);
                    }
                }
            } else {
#pragma unroll
                for (int d = 0; d < kQe; ++d)
                    x[d] = rv ? __uint_as_float(static_cast<uint32_t>(__ldg(src + d * p.qs3)) << 16) : 0.0f;
            }
            // stages h = 1 .. D / 8 inside the quarter
#pragma unroll
            for (int lg = 0; lg < kLgQe; ++lg) {
                const int hh = 1 << lg;
#pragma unroll
                for (int kk = 0; kk < kQe / 2; ++kk) {
                    const int j = ((kk >> lg) << (lg + 1)) + (kk & (hh - 1));
                    const float a = x[j], c = x[j + hh];
                    x[j] = __fadd_rn(a, c);
                    x[j + hh] = __fsub_rn(a, c);
                }
            }
            // stages h = D / 4 and D / 2 across the row's threads: x[j] +- x[j + h]
#pragma unroll
            for (int st = 1; st <= 2; st <<= 1) {
                const bool upper = (qq & st) != 0;
#pragma unroll
                for (int j = 0; j < kQe; ++j) {
                    const float y = __shfl_xor_sync(0xffffffffu, x[j], st);
                    x[j] = upper ? __fsub_rn(y, x[j]) : __fadd_rn(x[j], y);
                }
            }
            float amax = 0.0f;
#pragma unroll
            for (int d = 0; d < kQe; ++d) amax = fmaxf(amax, fabsf(x[d]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            float s = 0.0f, rr = 0.0f;
            if (amax != 0.0f) {
                s = __fdiv_rn(amax, 448.0f);
                rr = __fdiv_rn(448.0f, amax);
            }
            if (qq == 0) sq[r] = s;
            // the codes and scale also go to the caller's optional outputs
            // (written once, by the first CTA of (b, hk))
            const bool qout = rv && r == rq && split == 0 && p.q8_out != nullptr;
            const int64_t qtok = ((int64_t)b * p.T + t) * p.H + h;
            if (rv && r == rq && split == 0 && qq == 0 && p.qs_out != nullptr) p.qs_out[qtok] = s;
            uint8_t* qrow = sm + Sm::kQ + r * kD;
#pragma unroll
            for (int c = 0; c < kD / 64; ++c) {      // 16-byte chunk (D / 64) qq + c of the row
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int d = 16 * c + 4 * e;
                    const uint32_t lo16 = e4m3x2_rn_satfinite(__fmul_rn(x[d], rr), __fmul_rn(x[d + 1], rr));
                    const uint32_t hi16 = e4m3x2_rn_satfinite(__fmul_rn(x[d + 2], rr), __fmul_rn(x[d + 3], rr));
                    w4[e] = amax != 0.0f ? (lo16 | (hi16 << 16)) : 0u;   // a zero row: +0 codes
                }
                const int chunk = (kD / 64) * qq + c;
                if constexpr (MX) {
                    // the codes' exact bf16 values (A of a bf16 QK), eight
                    // channels per 16-byte chunk in the order in which the
                    // converters lay out K: pair m = (channel m, m + 4)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int k8 = 2 * chunk + hh;
                        const uint32_t wa = w4[2 * hh], wb = w4[2 * hh + 1];
                        *reinterpret_cast<uint4*>(sm + Sm::kQ + (k8 >> 3) * (kRows * 128) + r * 128 +
                                                  (((k8 & 7) ^ (r & 7)) << 4)) =
                            make_uint4(e4m3_pick_to_bf16x2<0>(wa, wb), e4m3_pick_to_bf16x2<1>(wa, wb),
                                       e4m3_pick_to_bf16x2<2>(wa, wb), e4m3_pick_to_bf16x2<3>(wa, wb));
                    }
                } else {
                    *reinterpret_cast<uint4*>(qrow + (e4m3_chunk<D>(chunk, r) << 4)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                if (qout)
                    *reinterpret_cast<uint4*>(p.q8_out + qtok * kD + 16 * chunk) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            if constexpr (NREP > 1) {
                // a warp writes only its own key columns of P'; the others
                // of its rows stay zero
                uint4* pz = reinterpret_cast<uint4*>(sm + Sm::kP);
                for (int z = tid; z < 2 * Sm::kPBuf / 16; z += kSoftWarps * 32) pz[z] = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();                // the QK / PV MMAs read these rows
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Sm::kQReady]);
        named_sync(1, kSoftWarps * 32);              // every row's s_q is in shared memory

        // Group g = warp >> 2 takes the tiles i = g, g + 2, g + 4, ... with
        // its own running max and sum, accumulated into O[g]; the groups run
        // side by side and are combined after the last tile. Warp qw = warp &
        // 3 of a group holds A rows 16 qw .. 16 qw + 15 (TMEM lanes 32 qw ..)
        // over the 2 kNC columns that begin at cb: thread: row r, register k
        // = column cb + 2k + cpar (k = 0 .. kNC - 1).
        const int qw = warp & 3, g = warp >> 2;
        const int lr = (lane >> 2) + 8 * (lane & 1);
        const int cpar = (lane >> 1) & 1;
        const int r = 16 * qw + lr;
        const int rq = r % kPeriod;                       // its query row
        const int cb = (qw / (4 / NREP)) * (2 * kNC);
        const bool rv = rq < p.R;
        const int pq = rv ? ctx - p.T + rq / p.G : -1;    // the row's query position
        // base-2 logit of a key = (acc * k_scale) * cq; cq kept >= FLT_MIN so
        // that a masked key (-inf) times cq stays -inf (a zero query row has
        // acc = 0, so its logits are 0 either way)
        const float cq = fmaxf(rv ? sq[r] * p.logit_scale_log2 : 0.0f, FLT_MIN);
        const uint64_t cq2 = f2_pack(cq, cq);
        const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * qw) << 16);
        float m_run = -INFINITY;                      // the max O[g] and the sum are expressed against
        uint64_t lsum2 = f2_pack(0.0f, 0.0f);         // running sum as an f32x2 pair
        bool ok = true;
        const int nt_mine = (NREP > 1 || 16 * qw < p.R) ? nt : 0;   // a warp of padding rows only sits out
        for (int i = g; i < nt_mine; i += 2) {
            const int c = i % kScStages;
            ok = warp_all(mbar_wait(&bars[Sm::kSFull + g], (i >> 1) & 1, abort_flag, &g_decode_err, 5));
            if (ok)
                ok = warp_all(mbar_wait(&bars[Sm::kScFull + c], (i / kScStages) & 1, abort_flag,
                                        &g_decode_err, 6));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[kNC];
            tmem_ld16_cols(taddr + 128 * g + cb, sv);

            const float* ksP = scl + c * kScSlot + cpar * kScPar + cb / 2;   // k_scale of column cb + 2k + cpar
            const float* vsP = ksP + kScHalf;
            const int key0 = (tb + i) * kKeys;
            const int kc0 = key0 + cb;                  // the key of register 0 (cpar 0)
            const int badm = meta[c];
            // y = acc * k_scale; the logit is y * cq, and cq > 0 keeps the
            // order, so the row max is taken on y
            float x[kNC];
#pragma unroll
            for (int k4 = 0; k4 < kNC / 4; ++k4) {
                const float4 kq = *reinterpret_cast<const float4*>(ksP + 4 * k4);
                const uint64_t a01 = f2_mul(f2_pack(__uint_as_float(sv[4 * k4]), __uint_as_float(sv[4 * k4 + 1])),
                                            f2_pack(kq.x, kq.y));
                const uint64_t a23 = f2_mul(f2_pack(__uint_as_float(sv[4 * k4 + 2]), __uint_as_float(sv[4 * k4 + 3])),
                                            f2_pack(kq.z, kq.w));
                f2_unpack(a01, x[4 * k4], x[4 * k4 + 1]);
                f2_unpack(a23, x[4 * k4 + 2], x[4 * k4 + 3]);
            }
            // masks: rows past R; keys outside the row's window; bad pages.
            // A tile inside every row's window with no bad page needs none.
            const bool full = badm == 0 && key0 >= ctx - p.window && key0 + kKeys - 1 <= ctx - p.T;
            if (!rv) {
#pragma unroll
                for (int k = 0; k < kNC; ++k) x[k] = -INFINITY;
            } else if (!full) {
                // the row sees keys [kc0 + clo, kc0 + chi] of this thread's
                const int clo = pq - p.window + 1 - kc0 - cpar, chi = pq - kc0 - cpar;
#pragma unroll
                for (int k = 0; k < kNC; ++k) x[k] = (2 * k >= clo && 2 * k <= chi) ? x[k] : -INFINITY;
                if (badm != 0) {
#pragma unroll
                    for (int k = 0; k < kNC; ++k)
                        if ((badm >> ((cb + 2 * k + cpar) >> p.lg_page)) & 1) x[k] = -INFINITY;
                }
            }
            // row max: four chains, a tree, the column partner
            float m4[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) m4[q4] = fmax3(x[q4], x[q4 + 4], x[q4 + 8]);
#pragma unroll
            for (int k = 12; k + 8 <= kNC - 4; k += 8)
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) m4[q4] = fmax3(m4[q4], x[k + q4], x[k + q4 + 4]);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) m4[q4] = fmaxf(m4[q4], x[kNC - 4 + q4]);
            float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mx = mx == -INFINITY ? -INFINITY : mx * cq;   // the max of the logits y * cq
            const float m_new = fmaxf(m_run, mx);
            // O[g] and the sum (tiles i - 2, i - 4, ...) are brought to m_new
            const bool resc = m_run != -INFINITY && m_new != m_run;
            const float alpha = resc ? ex2_approx(m_run - m_new) : 1.0f;
            if (resc) lsum2 = f2_mul(lsum2, f2_pack(alpha, alpha));
            m_run = m_new;
            const float sub = m_new == -INFINITY ? 0.0f : m_new;
            const uint64_t nsub2 = f2_pack(-sub, -sub);

            // P' buffer g and O[g] are free once PV(i - 2) is done
            if (i >= 2) {
                ok = warp_all(mbar_wait(&bars[Sm::kPvDone + g], ((i - 2) >> 1) & 1, abort_flag,
                                        &g_decode_err, 15));
                if (!ok) break;
                tc_fence_after();
            }
            uint8_t* prow = sm + Sm::kP + g * Sm::kPBuf + r * 128;
#pragma unroll
            for (int i16 = 0; i16 < kNC / 8; ++i16) {   // keys cb + 16 i16 + cpar + 2m = registers 8 i16 + m
                const float4 va = *reinterpret_cast<const float4*>(vsP + 8 * i16);
                const float4 vb = *reinterpret_cast<const float4*>(vsP + 8 * i16 + 4);
                const float vsv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
                uint32_t wd[4];
#pragma unroll
                for (int m = 0; m < 8; m += 2) {
                    float e0, e1;
                    f2_unpack(f2_fma(f2_pack(x[8 * i16 + m], x[8 * i16 + m + 1]), cq2, nsub2), e0, e1);
                    const float p0 = ex2_approx(e0), p1 = ex2_approx(e1);
                    const uint64_t p2 = f2_pack(p0, p1);
                    lsum2 = f2_add(lsum2, p2);
                    float w0, w1;
                    f2_unpack(f2_mul(p2, f2_pack(vsv[m], vsv[m + 1])), w0, w1);
                    const __nv_bfloat162 pr = __floats2bfloat162_rn(w0, w1);
                    wd[m / 2] = *reinterpret_cast<const uint32_t*>(&pr);
                }
                const int kb = cb / 16 + i16;            // 16-key block of the tile
                const int chunk = 2 * (kb & 3) + cpar;
                *reinterpret_cast<uint4*>(prow + (kb >> 2) * (kRows * 128) + ((chunk ^ (r & 7)) << 4)) =
                    make_uint4(wd[0], wd[1], wd[2], wd[3]);
            }
            // O[g] *= alpha for the rows whose max rose (PV(i - 2), its last
            // writer, is done), 64 columns at a time
            if (__any_sync(0xffffffffu, resc)) {
                tc_fence_after();
#pragma unroll
                for (int hf = 0; hf < kD / 64; ++hf) {
                    uint32_t o[32];
                    tmem_ld16x32(taddr + kOCol + kD * g + 64 * hf, o);
                    tmem_wait_ld(o);
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                    tmem_st16x32(taddr + kOCol + kD * g + 64 * hf, o);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();               // P' is read by the PV MMAs
            tc_fence_before();                      // S(i) read: QK(i + 2) may overwrite it
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[Sm::kPReady + g]);
                mbar_arrive(&bars[Sm::kScEmpty + c]);
            }
        }
        // the group's (m, l) per row, for the combination of O[0] and O[1]
        {
            float l0, l1;
            f2_unpack(lsum2, l0, l1);
            float lsum = l0 + l1;
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
            float* grp = reinterpret_cast<float*>(sm + Sm::kGrp);
            if (cpar == 0) {
                grp[g * kRows + r] = ok ? m_run : -INFINITY;
                grp[2 * kRows + g * kRows + r] = ok ? lsum : 0.0f;
            }
        }
        named_sync(1, kSoftWarps * 32);
        // this warp's output channels: 64 g .. 64 g + 63 of its rows;
        // O = O[0] 2^(m0 - M) + O[1] 2^(m1 - M), l likewise, M = max(m0, m1)
        float o_fin[kOe];
        float m_fin = -INFINITY, l_fin = 0.0f;
        bool have = nt > 0 && warp_all(mbar_wait(&bars[Sm::kPvDone + ((nt - 1) & 1)], ((nt - 1) >> 1) & 1,
                                                 abort_flag, &g_decode_err, 9));
#pragma unroll
        for (int k = 0; k < kOe; ++k) o_fin[k] = 0.0f;
        if (have) {
            // (the TMEM loads are warp-wide: every lane takes them, and a row
            // whose group saw no key, m = -inf, takes none of their values)
            const float* grp = reinterpret_cast<const float*>(sm + Sm::kGrp);
            const float m0 = grp[r], m1 = grp[kRows + r];
            m_fin = fmaxf(m0, m1);
            tc_fence_after();
            {
                const bool use0 = m0 != -INFINITY;
                const float w0 = use0 ? ex2_approx(m0 - m_fin) : 0.0f;
                uint32_t o0[kOe];
                tmem_ld16_wait(taddr + kOCol + (kD / 2) * g, o0);
#pragma unroll
                for (int k = 0; k < kOe; ++k) o_fin[k] = use0 ? __uint_as_float(o0[k]) * w0 : 0.0f;
                l_fin = use0 ? grp[2 * kRows + r] * w0 : 0.0f;
            }
            if (nt > 1) {
                const bool use1 = m1 != -INFINITY;
                const float w1 = use1 ? ex2_approx(m1 - m_fin) : 0.0f;
                uint32_t o1[kOe];
                tmem_ld16_wait(taddr + kOCol + kD + (kD / 2) * g, o1);
#pragma unroll
                for (int k = 0; k < kOe; ++k)
                    o_fin[k] = use1 ? fmaf(__uint_as_float(o1[k]), w1, o_fin[k]) : o_fin[k];
                if (use1) l_fin = fmaf(grp[3 * kRows + r], w1, l_fin);
            }
        }
        // ---- the CTA's (m, l, O) per row, staged row-major over the K stages
        // (free once every role is past the CTA barrier): the output itself
        // when the CTA holds every tile of (b, hk), else a partial in the
        // workspace that the merge kernel combines
        tc_fence_before();
        bar_sync_all(kThreads);
        {
            float* oc = reinterpret_cast<float*>(sm + Sm::kOc);
            float2* stat = reinterpret_cast<float2*>(sm + Sm::kStat);
            // (MX: TMEM column 8 u + 2 m + c holds channel 8 u + m + 4 c, the
            // order of the converted V rows)
#pragma unroll
            for (int k = 0; k < kOe; ++k)
                oc[r * kOcPitch + (kD / 2) * g + (MX ? 8 * (k >> 2) + (k & 3) + 4 * cpar : 2 * k + cpar)] = o_fin[k];
            if (g == 0 && cpar == 0) stat[r] = make_float2(m_fin, l_fin);
            named_sync(1, kSoftWarps * 32);
            // query row rr: its NREP A rows rr + u kPeriod combined
            auto row_stat = [&](int rr) -> float2 {
                if constexpr (NREP == 1) {
                    return stat[rr];
                } else {
                    float M = -INFINITY, L = 0.0f;
#pragma unroll
                    for (int u = 0; u < NREP; ++u) M = fmaxf(M, stat[rr + u * kPeriod].x);
#pragma unroll
                    for (int u = 0; u < NREP; ++u) {
                        const float2 su = stat[rr + u * kPeriod];
                        if (su.x != -INFINITY) L = fmaf(ex2_approx(su.x - M), su.y, L);
                    }
                    return make_float2(M, L);
                }
            };
            auto row_o4 = [&](int rr, int d4, float M) -> float4 {
                if constexpr (NREP == 1) {
                    return *reinterpret_cast<const float4*>(oc + rr * kOcPitch + d4);
                } else {
                    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
                    for (int u = 0; u < NREP; ++u) {
                        const float mu = stat[rr + u * kPeriod].x;
                        if (mu == -INFINITY) continue;
                        const float w = ex2_approx(mu - M);
                        const float4 o = *reinterpret_cast<const float4*>(oc + (rr + u * kPeriod) * kOcPitch + d4);
                        acc.x = fmaf(w, o.x, acc.x);
                        acc.y = fmaf(w, o.y, acc.y);
                        acc.z = fmaf(w, o.z, acc.z);
                        acc.w = fmaf(w, o.w, acc.w);
                    }
                    return acc;
                }
            };
            if (p.nsplit == 1) {
                // thread: one row, four channels
                for (int idx = tid; idx < p.R * (kD / 4); idx += kSoftWarps * 32) {
                    const int rr = idx / (kD / 4), d4 = 4 * (idx % (kD / 4));
                    const float2 st = row_stat(rr);
                    store_out4(p, b, hk, rr, d4, row_o4(rr, d4, st.x), st.y > 0.0f ? 1.0f / st.y : 0.0f);
                }
            } else {
                // the partial to the workspace, combined by decode_merge_kernel
                const size_t part = (size_t)bhk * p.nsplit + split;
                float4* wo = reinterpret_cast<float4*>(p.ws_o + part * kRows * kD);
                for (int idx = tid; idx < p.R * (kD / 4); idx += kSoftWarps * 32) {
                    const int rr = idx / (kD / 4), d4 = 4 * (idx % (kD / 4));
                    wo[idx] = row_o4(rr, d4, row_stat(rr).x);
                }
                if (tid < p.R) p.ws_stat[part * kRows + tid] = row_stat(tid);
            }
        }
    } else {
      reg_dealloc<RegSplit<MX, NREP>::conv>();
        // ------------------------------------------------------------ V converters
        // lane -> V row kap of the tile (warp cw: rows 32 cw .. 32 cw + 31),
        // chosen so that the eight lanes of a quarter-warp read eight
        // different 16-byte bank groups and write eight different ones
        const int cw = warp - kConvWarp0;
        const int q8 = lane >> 3, e8 = lane & 7;
        const int kap = 32 * cw + 16 * (q8 >> 1) + 2 * e8 + ((e8 >> 2) ^ (q8 & 1));
        const int pos = pv_position(kap);
        bool ok = true;
        if constexpr (MX) {
        // MX: K(i) to the one bf16 K buffer (once QK(i - 1) has read it),
        // lane -> key 32 cw + lane in key order; then V(i) to bf16 buffer
        // i & 1 as below. A code row is 64 bytes (64B-swizzled by the TMA),
        // one 16-byte chunk per 32-channel block, its e8m0 scales 4 bytes.
        for (int i = 0; i < nt; ++i) {
            const int s = i % kStages, bf = i & 1;
            ok = warp_all(mbar_wait(&bars[Sm::kKvFull + s], (i / kStages) & 1, abort_flag, &g_decode_err, 10));
            if (ok && i >= 1)
                ok = warp_all(mbar_wait(&bars[Sm::kKbFree], (i - 1) & 1, abort_flag, &g_decode_err, 16));
            if (!ok) break;
            {
                const int key = 32 * cw + lane;
                const uint8_t* krow = sm + Sm::kK + s * Sm::kKStage + key * 64;
                const uint32_t esc = *reinterpret_cast<const uint32_t*>(sm + Sm::kKsf + s * Sm::kSfStage + key * 4);
                uint8_t* dst = sm + Sm::kKb + key * 128;
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t o[16];
                    e2m1_block_to_bf16(*reinterpret_cast<const uint4*>(krow + (e4m3_chunk<64>(blk, key) << 4)),
                                       (esc >> (8 * blk)) & 0xFFu, o);
                    uint8_t* atom = dst + (blk >> 1) * (kKeys * 128);
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq)
                        *reinterpret_cast<uint4*>(atom + (((4 * (blk & 1) + gq) ^ (key & 7)) << 4)) =
                            make_uint4(o[4 * gq], o[4 * gq + 1], o[4 * gq + 2], o[4 * gq + 3]);
                }
            }
            fence_proxy_async_smem();               // read by the QK MMAs
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[Sm::kKbReady]);
            if (i >= 2)
                ok = warp_all(mbar_wait(&bars[Sm::kPvDone + bf], ((i - 2) >> 1) & 1, abort_flag,
                                        &g_decode_err, 11));
            if (!ok) break;
            {
                const uint8_t* vrow = sm + Sm::kV + s * Sm::kKStage + kap * 64;
                const uint32_t esc = *reinterpret_cast<const uint32_t*>(sm + Sm::kVsf + s * Sm::kSfStage + kap * 4);
                uint8_t* dst = sm + Sm::kVb + bf * Sm::kVbBuf + pos * 128;
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t o[16];
                    e2m1_block_to_bf16(*reinterpret_cast<const uint4*>(vrow + (e4m3_chunk<64>(blk, kap) << 4)),
                                       (esc >> (8 * blk)) & 0xFFu, o);
                    uint8_t* atom = dst + (blk >> 1) * (kKeys * 128);
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq)
                        *reinterpret_cast<uint4*>(atom + (((4 * (blk & 1) + gq) ^ (pos & 7)) << 4)) =
                            make_uint4(o[4 * gq], o[4 * gq + 1], o[4 * gq + 2], o[4 * gq + 3]);
                }
            }
            fence_proxy_async_smem();               // read by the PV MMAs
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[Sm::kPReady + bf]);
                mbar_arrive(&bars[Sm::kKvEmpty + s]);
            }
        }
        } else {
        for (int i = 0; i < nt; ++i) {
            const int s = i % kStages, bf = i & 1;
            ok = warp_all(mbar_wait(&bars[Sm::kKvFull + s], (i / kStages) & 1, abort_flag, &g_decode_err, 10));
            if (ok && i >= 2)
                ok = warp_all(mbar_wait(&bars[Sm::kPvDone + bf], ((i - 2) >> 1) & 1, abort_flag,
                                        &g_decode_err, 11));
            if (!ok) break;
            if (p.v_trans) {
                // V^T tile [D channels][128 keys]: lane -> channel row d; its
                // keys become the row of a K-major bf16 operand in the key order
                // of P' (per 16 keys: the even keys, then the odd ones)
                const int d = 32 * cw + lane;
                const uint8_t* vrow = sm + Sm::kV + s * Sm::kKStage + d * 128;
                uint8_t* dst = sm + Sm::kVb + bf * Sm::kVbBuf + d * 128;
#pragma unroll
                for (int c = 0; c < 8 && d < kD; ++c) {   // keys 16c .. 16c + 15
                    const uint4 u = *reinterpret_cast<const uint4*>(vrow + ((c ^ (d & 7)) << 4));
                    const uint32_t e0 = e4m3x2_to_bf16x2(u.x, 0x2404u), e1 = e4m3x2_to_bf16x2(u.y, 0x2404u);
                    const uint32_t e2 = e4m3x2_to_bf16x2(u.z, 0x2404u), e3 = e4m3x2_to_bf16x2(u.w, 0x2404u);
                    const uint32_t d0 = e4m3x2_to_bf16x2(u.x, 0x3414u), d1 = e4m3x2_to_bf16x2(u.y, 0x3414u);
                    const uint32_t d2 = e4m3x2_to_bf16x2(u.z, 0x3414u), d3 = e4m3x2_to_bf16x2(u.w, 0x3414u);
                    uint8_t* atom = dst + (c >> 2) * (kD * 128);
                    const int g2 = 2 * (c & 3);
                    *reinterpret_cast<uint4*>(atom + ((g2 ^ (d & 7)) << 4)) = make_uint4(e0, e1, e2, e3);
                    *reinterpret_cast<uint4*>(atom + (((g2 + 1) ^ (d & 7)) << 4)) = make_uint4(d0, d1, d2, d3);
                }
            } else {
            const uint8_t* vrow = sm + Sm::kV + s * Sm::kKStage + kap * kD;
            uint8_t* dst = sm + Sm::kVb + bf * Sm::kVbBuf + pos * 128;
#pragma unroll
            for (int c = 0; c < kD / 16; ++c) {     // channels 16c .. 16c + 15
                const uint4 u = *reinterpret_cast<const uint4*>(vrow + (e4m3_chunk<D>(c, kap) << 4));
                const uint32_t o0 = e4m3x2_to_bf16x2(u.x, 0x1404u), o1 = e4m3x2_to_bf16x2(u.x, 0x3424u);
                const uint32_t o2 = e4m3x2_to_bf16x2(u.y, 0x1404u), o3 = e4m3x2_to_bf16x2(u.y, 0x3424u);
                const uint32_t o4 = e4m3x2_to_bf16x2(u.z, 0x1404u), o5 = e4m3x2_to_bf16x2(u.z, 0x3424u);
                const uint32_t o6 = e4m3x2_to_bf16x2(u.w, 0x1404u), o7 = e4m3x2_to_bf16x2(u.w, 0x3424u);
                uint8_t* half = dst + (c >> 2) * (kKeys * 128);
                const int ch = 2 * (c & 3);
                *reinterpret_cast<uint4*>(half + ((ch ^ (pos & 7)) << 4)) = make_uint4(o0, o1, o2, o3);
                *reinterpret_cast<uint4*>(half + (((ch + 1) ^ (pos & 7)) << 4)) = make_uint4(o4, o5, o6, o7);
            }
            }
            fence_proxy_async_smem();               // read by the PV MMAs
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[Sm::kPReady + bf]);
                mbar_arrive(&bars[Sm::kKvEmpty + s]);
            }
        }
        }
        tc_fence_before();
        bar_sync_all(kThreads);
    }
}

// The splits of (b, hk) combined (log-sum-exp): thread = one query row and
// four channels; every split's (m, l) and O loaded before any use.
template <int D>
__global__ void __launch_bounds__(256) decode_merge_kernel(const DecParams p) {
    pdl_launch_dependents();                 // the next decode may start its setup
    const int bhk = blockIdx.x, hk = bhk % p.Hk, b = bhk / p.Hk;
    const int idx = blockIdx.y * 256 + threadIdx.x;
    const int rr = idx / (D / 4), d4 = 4 * (idx % (D / 4));
    if (rr >= p.R) return;
    const size_t part0 = (size_t)bhk * p.nsplit;
    float2 st[kMaxSplit];
    float4 ov[kMaxSplit];
#pragma unroll
    for (int sp = 0; sp < kMaxSplit; ++sp) {
        if (sp < p.nsplit) {
            st[sp] = __ldcg(p.ws_stat + (part0 + sp) * kRows + rr);
            ov[sp] = __ldcg(reinterpret_cast<const float4*>(p.ws_o + ((part0 + sp) * kRows + rr) * D + d4));
        } else {
            st[sp] = make_float2(-INFINITY, 0.0f);
            ov[sp] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
    }
    float M = -INFINITY;
#pragma unroll
    for (int sp = 0; sp < kMaxSplit; ++sp) M = fmaxf(M, st[sp].x);
    float den = 0.0f;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (M != -INFINITY) {
#pragma unroll
        for (int sp = 0; sp < kMaxSplit; ++sp) {
            const float wgt = st[sp].x == -INFINITY ? 0.0f : ex2_approx(st[sp].x - M);
            den = fmaf(wgt, st[sp].y, den);
            acc.x = fmaf(wgt, ov[sp].x, acc.x);
            acc.y = fmaf(wgt, ov[sp].y, acc.y);
            acc.z = fmaf(wgt, ov[sp].z, acc.z);
            acc.w = fmaf(wgt, ov[sp].w, acc.w);
        }
    }
    store_out4(p, b, hk, rr, d4, acc, den > 0.0f ? 1.0f / den : 0.0f);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The cache [num_pages, Hk, page, D] e4m3 as a 3-D map {D bytes, page
// rows, num_pages * Hk}; one box = one page of one kv head, with the swizzle
// of a D-byte row (128B or 64B).
bool encode_cache(CUtensorMap* map, const void* ptr, int num_pages, int Hk, int page, int D) {
    auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(page),
                                static_cast<cuuint64_t>(num_pages) * Hk};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(page) * D};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(page), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The transposed V cache [num_pages, Hk, D, page = 128] as a 3-D map
// {128 key bytes, D channel rows, num_pages * Hk}; one box = one page of
// one kv head as [channel][key], 128B swizzle.
bool encode_cache_vt(CUtensorMap* map, const void* ptr, int num_pages, int Hk, int D) {
    auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kKeys), static_cast<cuuint64_t>(D),
                                static_cast<cuuint64_t>(num_pages) * Hk};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kKeys), static_cast<cuuint64_t>(D) * kKeys};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kKeys), static_cast<cuuint32_t>(D), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The MXFP4 cache codes [num_pages, Hk, page, D / 2] bytes (two E2M1 codes a
// byte) as a 3-D map {D / 2 bytes, page rows, num_pages * Hk}; one box = one
// page of one kv head, 64B swizzle (D = 128: 64-byte rows).
bool encode_cache_mx(CUtensorMap* map, const void* ptr, int num_pages, int Hk, int page, int D) {
    auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!enc || D != 128) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D / 2), static_cast<cuuint64_t>(page),
                                static_cast<cuuint64_t>(num_pages) * Hk};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D / 2), static_cast<cuuint64_t>(page) * (D / 2)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(D / 2), static_cast<cuuint32_t>(page), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool MX>
constexpr int smem_bytes() { return SmL<D, MX>::kBytes + 1024; }

// Repeats of the query rows in the QK A operand for R query rows.
int pick_nrep(int R) { return R <= 16 ? 4 : (R <= 32 ? 2 : 1); }

// Streaming multiprocessors of the current device (queried once per device).
int device_sms() {
    static std::mutex mu;
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
    std::lock_guard<std::mutex> lock(mu);
    int& c = cache[dev];
    if (c == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = 1;
        }
        c = n;
    }
    return c;
}

// The most CTAs per (sequence, kv head): a split grid stays within one wave
// (one CTA per SM), so that it and the merge are all the work there is.
int max_split(int n_seq_heads) {
    return std::max(1, std::min(kMaxSplit, device_sms() / std::max(1, n_seq_heads)));
}

// CTAs per (sequence, kv head): the one that minimises the most 128-key
// tiles a CTA gets (for the most tiles a sequence can span) plus the merge,
// counted as half a tile; of equal choices the smaller.
int pick_nsplit(int n_seq_heads, int T, int window, int page, int max_pages) {
    const int64_t span = std::min<int64_t>((int64_t)window + T - 1, (int64_t)max_pages * page);
    const int64_t tiles = std::max<int64_t>(1, ceil_div(span, kKeys) + 1);
    const int cap = max_split(n_seq_heads);
    int best = 1;
    int64_t best_cost = INT64_MAX;
    for (int sz = 1; sz <= std::min<int64_t>(cap, tiles); ++sz) {
        const int64_t cost = 2 * ceil_div(tiles, sz) + (sz > 1 ? 1 : 0);
        if (cost < best_cost) {
            best_cost = cost;
            best = sz;
        }
    }
    return best;
}

}  // namespace

// Partials for the most splits the launch may pick: (m, l) and O per row.
size_t decode_ws_bytes(int B, int, int, int Hk, int D, int) {
    const int cap = max_split(B * Hk);
    if (cap <= 1) return 0;
    return (size_t)B * Hk * cap * kRows * (sizeof(float2) + D * sizeof(float));
}

namespace {

template <int D, bool MX>
cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t s) {
    constexpr int kSmemBytes = smem_bytes<D, MX>();
    DecParams p;
    p.q = static_cast<const uint16_t*>(a.q.ptr);
    p.qs0 = a.q.stride[0];
    p.qs1 = a.q.stride[1];
    p.qs2 = a.q.stride[2];
    p.qs3 = a.q.stride[3];
    p.ksc = a.k_scale;
    p.vsc = a.v_scale;
    p.ptab = a.page_table;
    p.ctx = a.ctx_lens;
    p.T = a.T;
    p.H = a.H;
    p.Hk = a.Hk;
    p.G = a.H / a.Hk;
    p.R = a.T * p.G;
    p.page = a.page_size;
    p.lg_page = 31 - __builtin_clz(static_cast<unsigned>(a.page_size));
    p.max_pages = a.max_pages;
    p.num_pages = a.num_pages;
    p.window = a.window;
    p.logit_scale_log2 = a.softmax_scale / static_cast<float>(a.D) * kLog2e;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.os0 = a.out_stride[0];
    p.os1 = a.out_stride[1];
    p.os2 = a.out_stride[2];
    p.os3 = a.out_stride[3];
    p.q8_out = a.q8_out;
    p.qs_out = a.q_scale_out;
    p.per_tensor = (a.kv_flags & 1) ? 1 : 0;
    p.v_trans = (!MX && (a.kv_flags & 2)) ? 1 : 0;
    p.ksf8 = a.k_sf;
    p.vsf8 = a.v_sf;
    p.q_vec = (a.q.stride[3] == 1 && a.q.stride[0] % 8 == 0 && a.q.stride[1] % 8 == 0 &&
               a.q.stride[2] % 8 == 0 && reinterpret_cast<uintptr_t>(a.q.ptr) % 16 == 0)
                  ? 1
                  : 0;
    CUtensorMap tk, tv;
    if (MX) {
        if (!encode_cache_mx(&tk, a.k_cache, a.num_pages, a.Hk, a.page_size, D) ||
            !encode_cache_mx(&tv, a.v_cache, a.num_pages, a.Hk, a.page_size, D))
            return cudaErrorInvalidValue;
    } else if (!encode_cache(&tk, a.k_cache, a.num_pages, a.Hk, a.page_size, D) ||
               !(p.v_trans ? encode_cache_vt(&tv, a.v_cache, a.num_pages, a.Hk, D)
                           : encode_cache(&tv, a.v_cache, a.num_pages, a.Hk, a.page_size, D))) {
        return cudaErrorInvalidValue;
    }
    const int nrep = pick_nrep(p.R);
    auto kern = nrep == 4 ? decode_kernel<D, MX, 4> : (nrep == 2 ? decode_kernel<D, MX, 2> : decode_kernel<D, MX, 1>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    p.nsplit = pick_nsplit(a.B * a.Hk, a.T, a.window, a.page_size, a.max_pages);
    p.o_vec = (a.out_stride[3] == 1 && a.out_stride[0] % 4 == 0 && a.out_stride[1] % 4 == 0 &&
               a.out_stride[2] % 4 == 0 && reinterpret_cast<uintptr_t>(a.out) % 8 == 0)
                  ? 1
                  : 0;
    p.ws_stat = nullptr;
    p.ws_o = nullptr;
    if (p.nsplit > 1) {
        if (a.ws == nullptr) return cudaErrorInvalidValue;
        p.ws_stat = static_cast<float2*>(a.ws);
        p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) +
                                          (size_t)a.B * a.Hk * p.nsplit * kRows * sizeof(float2));
    }
    // a programmatic dependent of whatever precedes it on the stream: only
    // the setup before griddepcontrol.wait overlaps that kernel
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.nsplit, a.B * a.Hk);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tk, tv, p);
    if (e != cudaSuccess || p.nsplit == 1) return e;
    // a plain stream-ordered launch: it measured faster here than one
    // launched as a programmatic dependent of the split grid
    decode_merge_kernel<D><<<dim3(a.B * a.Hk, (p.R * (D / 4) + 255) / 256), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    if (a.mx) return a.D == 128 ? launch_decode_d<128, true>(a, s) : cudaErrorInvalidValue;
    switch (a.D) {
        case 64: return launch_decode_d<64, false>(a, s);
        case 128: return launch_decode_d<128, false>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

unsigned read_clear_decode_error() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_decode_err, sizeof v) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_decode_err, &zero, sizeof zero);
    return v;
}

}  // namespace sage
