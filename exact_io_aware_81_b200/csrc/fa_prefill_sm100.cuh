// fa_prefill_sm100.cuh -- exact attention forward (prefill) for sm_100a.
//
// Method (youngju.dev "attention variants", section 3 FlashAttention; toolsku.com,
// generation 4): Q, K and V are cut into 128-row tiles that are staged into shared memory;
// for each query tile the key/value tiles are visited in order, a block of scores is
// formed on chip, and the softmax is accumulated online (running row maximum, running
// sum, rescale of the partial output when the maximum moves).  Only O and the row
// log-sum-exp go back to HBM; the (N, N) score matrix never exists in memory.  Causal
// masks skip key tiles wholly in the future, mask the tiles that cross the diagonal and
// compute the others in full (youngju.dev section 5.5).  Grouped-query heads share each
// staged key/value tile (youngju.dev section 2; toolsku.com generation 2).
//
// B200 mapping (one persistent CTA per SM, 12 warps = 3 warpgroups):
//   warp 8      TMA producer: Q tiles once per work unit into one of two Q buffers (the
//               next unit's Q loads while this one runs), K_j / V_j into an NSTAGE ring
//               of 128-byte-swizzled tiles, completion counted on mbarriers (the warp
//               runs the loop, one elected lane issues).
//   warp 9      MMA issuer (warp runs the loop, one elected lane issues):
//               S_s = Q_s K_j^T (both operands from shared memory) and
//               O_s += P_s V_j (P from tensor memory, V from shared memory) with
//               tcgen05.mma; accumulators live in tensor memory (512 columns:
//               S0 | S1 | O0 | O1, P_s packed as bf16 over the first 64 columns of S_s).
//   warps 0-3   softmax for Q tile 0, warps 4-7 for Q tile 1 (one thread per row):
//               load S_s from TMEM, mask, row max, exp2 with the scale folded in
//               (p = 2^(s*scale*log2e - m)), lazy rescale (the reference maximum is only
//               moved when the new one exceeds it by more than 16 in log2 units; O_s is
//               then rescaled in TMEM by the same warp), P_s to TMEM as bf16, fp32 row
//               sum; at the end of a unit O_s / l and LSE are written out.
//   warps 10-11 idle (they complete the third warpgroup, which lends registers to the
//               softmax warpgroups through setmaxnreg).
// FP8 variant (Q, K, V in E4M3 with one scale per head; toolsku.com, FlashAttention
// generations table, FP8 among FA3's data types): S = Q K^T runs as a kind::f8f6f4 MMA on
// the E4M3 tiles, the head scales folded into the softmax scale; warps 10-11 widen each V
// tile to fp16 in shared memory (the hardware conversion, exact), so P V stays a
// kind::f16 MMA with P rounded to fp16 (the lazy threshold is 8, so P <= 2^8 fits fp16);
// the epilogue applies v_scale / l and stages O through the unit's Q slot in two rounds.
// The two Q tiles of a work unit share their key/value head: two query heads of one
// group (R even) or two consecutive row tiles of one head (otherwise).  Their MMAs are
// interleaved S0_j, PV1_{j-1}, S1_j, PV0_j -- continued across units -- so that the
// tensor core works on one tile while the softmax warps work on the other.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa_common.cuh"
#include "ptx_sm100.cuh"

namespace fa {

struct PrefillParams {
    // The maps view every tensor as 4-D (d, rows, heads, batch) whatever its layout in memory
    // ((B, H, N, d) or (B, N, H, d)): only the strides differ.
    CUtensorMap tm_q;  // (d, Nq, Hq, B) bf16, box (64, 128, 1, 1), 128B swizzle
    CUtensorMap tm_k;  // (d, Nk, Hkv, B)
    CUtensorMap tm_v;  // (d, Nk, Hkv, B)
    CUtensorMap tm_o;  // (d, Nq, Hq, B) bf16 output, box (64, 32, 1, 1), 128B swizzle: one warp's rows
    void *o;
    long long o_sb, o_sh, o_sn;  // fp32 output: element strides of batch, head and row
    float *lse;
    int B, Hq, Hkv, Nq, Nk;
    int R;           // Hq / Hkv
    int causal;
    int window;      // sliding window W (causal only): row i sees keys (i+Nk-Nq-W, i+Nk-Nq]; 0 = none
    int head_pair;   // 1: a unit = heads (2p, 2p+1) of one group on the same 128 rows
    int T;           // tile rows per head slot: 128-row tiles (head_pair) or 256-row pairs
    int P;           // slots per head slot: ceil(T/2) if causal (units paired), else T
    int n_slots;     // head slots * P
    float scale_log2;  // scale * log2(e)
    unsigned long long wait_limit_ns;
    int selftest_no_s_signal;  // timeout self-test: never signal a ready score tile
    const float *q_scale, *k_scale, *v_scale;  // FP8 variant: per-head dequantization scales
    long long debug_lse_offset;  // debug builds' bounds self-test: added to every LSE index (else 0)
};

namespace prefill {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 384;   // 3 warpgroups
// Registers per thread: 168 at launch (384 threads share the 64K register file).  With
// setmaxnreg the producer/MMA warpgroup keeps kRegsLow and each softmax warpgroup gets
// kRegsHigh; 128 * kRegsLow + 256 * kRegsHigh must not exceed 384 * 168.
constexpr int kRegsLow = 72;
constexpr int kRegsHigh = 216;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= 384 * 168, "register split exceeds the launch budget");
constexpr int kChunkBytes = 128 * 128;  // one 64-column (128-byte) slab of a 128-row tile
constexpr float kLazyThreshold = 16.0f;  // log2 units: rescale only past a factor of 2^16
constexpr float kLazyThresholdF16 = 8.0f;  // FP8 variant: P <= 2^8 must fit fp16
constexpr float kLn2 = 0.6931471805599453f;

template <int D, bool FP8 = false>
struct Cfg {
    static constexpr int kTileBytes = 128 * D * 2;             // a 16-bit 128-row tile
    static constexpr int kInTileBytes = FP8 ? 128 * D : kTileBytes;  // a Q, K or V tile as loaded
    // Q is double-buffered (two sets of the unit's two Q tiles) so the next unit's Q is
    // loaded while the current one runs; the K/V ring gets what is left of 227 KB.  FP8: K
    // and V alternate in an even ring (K in even stages, V in odd ones) and two fp16 tiles
    // hold the widened V.
    static constexpr int kStages = FP8 ? 4 : (D == 128) ? 3 : 8;
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = 4 * kInTileBytes;
    static constexpr int kV16Off = kKVOff + kStages * kInTileBytes;
    static constexpr int kBarOff = kV16Off + (FP8 ? 2 * kTileBytes : 0);
    // barriers: kv_full[S], kv_empty[S], q_full[2 sets][2], q_empty[2 sets][2], s_full[2],
    //           p_ready[2], o_done[2], o_free[2], teardown, p_half[2]; FP8: v16_full[2],
    //           v16_empty[2]
    static constexpr int kNumBars = 2 * kStages + 19 + (FP8 ? 4 : 0);
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 64 + 1024;  // + alignment slack
};

// A unit: two 128-row Q tiles (s = 0, 1) of one K/V group; tile s reads key tiles
// [a_s, n_s).  a0 <= a1 and n0 <= n1, and every key tile in [a0, n1) is read by at least
// one of the two.
struct Unit {
    int b, g, h0, h1, r0, r1, a0, a1, n0, n1;
};

// Work is dealt out in slots.  A slot belongs to one "head slot" (a head pair of one
// K/V group, or one head) and, for causal masks, holds two units: tile row T-1-i (the
// heaviest left) and tile row i (the lightest), so every slot costs the same and a plain
// round-robin over the persistent CTAs stays balanced.  Head slots are numbered with the
// heads of one K/V group adjacent and slots of one head slot consecutive, so the CTAs
// running at any moment share few K/V heads and their tiles are re-read from L2.
__device__ __forceinline__ int units_in_slot(const PrefillParams &p) { return p.causal ? 2 : 1; }

// WINDOW: the kernel variant for sliding-window attention (p.window > 0); without it
// a0 = a1 = 0 are compile-time constants and the plain causal code is unchanged.
template <bool WINDOW>
__device__ __forceinline__ bool decode_unit(const PrefillParams &p, int slot, int k, Unit &w)
{
    const int hh = slot / p.P;
    const int pi = slot - hh * p.P;
    int t = pi;
    if (p.causal) {
        t = (k == 0) ? (p.T - 1 - pi) : pi;
        if (k == 1 && pi == p.T - 1 - pi) return false;  // middle tile row of an odd T
    }
    if (p.head_pair) {
        const int hpairs = p.R >> 1;
        const int hp = hh % hpairs;
        const int bg = hh / hpairs;
        w.g = bg % p.Hkv;
        w.b = bg / p.Hkv;
        w.h0 = w.g * p.R + 2 * hp;
        w.h1 = w.h0 + 1;
        w.r0 = w.r1 = BM * t;
    } else {
        const int h = hh % p.Hq;
        w.b = hh / p.Hq;
        w.g = h / p.R;
        w.h0 = w.h1 = h;
        w.r0 = 2 * BM * t;
        w.r1 = w.r0 + BM;
    }
    const int nkt = (p.Nk + BN - 1) / BN;
    w.a0 = w.a1 = 0;
    if (p.causal) {
        const int delta = p.Nk - p.Nq;
        // the last row of a tile, r + 127, sees keys up to r + 127 + delta
        w.n0 = min(nkt, (w.r0 + BM - 1 + delta) / BN + 1);
        w.n1 = min(nkt, (w.r1 + BM - 1 + delta) / BN + 1);
        if (WINDOW) {
            // the first row of a tile, r, sees keys from r + delta - W + 1 on
            w.a0 = max(0, w.r0 + delta - p.window + 1) / BN;
            w.a1 = max(0, w.r1 + delta - p.window + 1) / BN;
            // The second tile of a row pair can lie wholly past Nq (odd tile count) and
            // then past every window: its rows are never stored, so it reads only the
            // last key tile.  (Every other tile has a_s < n_s: its first row sees at
            // least its own diagonal key.)
            if (w.r1 >= p.Nq) w.a1 = w.n1 - 1;
        }
    } else {
        w.n0 = w.n1 = nkt;
    }
    return true;
}

// The units of this CTA in order: slots blockIdx.x, blockIdx.x + gridDim.x, ... and, inside
// a slot, its units k = 0, 1.  Unit index u = 2 * slot + k.
__device__ __forceinline__ int unit_step(int u) { return u + ((u & 1) ? 2 * (int)gridDim.x - 1 : 1); }

// First valid unit index >= u of this CTA (decoded into w), or -1.
template <bool WINDOW>
__device__ __forceinline__ int next_unit(const PrefillParams &p, int u, Unit &w)
{
    for (; u < 2 * p.n_slots; u = unit_step(u))
        if ((u & 1) < units_in_slot(p) && decode_unit<WINDOW>(p, u >> 1, u & 1, w)) return u;
    return -1;
}

// S = Q K^T over the full head dimension: D/16 MMAs of K = 16.  Both operands are
// K-major 128-byte-swizzled tiles: 8-row groups 1024 bytes apart (stride offset), a
// K step of 16 elements advances the start address by 32 bytes inside the swizzle
// atom, and the second 64-column slab (D = 128) starts 16 KB further on.  The start
// address is the descriptor's low field (address >> 4, 14 bits); shared-memory addresses
// stay below 256 KB, so adding (offset >> 4) to the base descriptor advances it exactly.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_saddr, uint32_t k_saddr)
{
    constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, BN, 0);
    const uint64_t a0 = ptx::smem_desc_sw128(q_saddr, 16, 1024);
    const uint64_t b0 = ptx::smem_desc_sw128(k_saddr, 16, 1024);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
        const uint64_t off = (uint64_t)(((k >> 2) * kChunkBytes + (k & 3) * 32) >> 4);
        ptx::mma_ss(d_tmem, a0 + off, b0 + off, idesc, k > 0 ? 1u : 0u);
    }
}

// FP8: S = Q K^T from E4M3 tiles, one 128-byte slab each (d = 128): 4 MMAs of K = 32.
__device__ __forceinline__ void issue_qk_fp8(uint32_t d_tmem, uint32_t q_saddr, uint32_t k_saddr)
{
    constexpr uint32_t idesc = ptx::idesc_f32acc(BM, BN, 0, 0, 0);  // E4M3 x E4M3
    const uint64_t a0 = ptx::smem_desc_sw128(q_saddr, 16, 1024);
    const uint64_t b0 = ptx::smem_desc_sw128(k_saddr, 16, 1024);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        ptx::mma_ss_f8(d_tmem, a0 + (uint64_t)(k * 2), b0 + (uint64_t)(k * 2), idesc, k > 0 ? 1u : 0u);
}

// O (+)= P V for K steps [k_begin, k_end) of the 8 (16 keys each).  P (128 x 128 bf16)
// is read from tensor memory, 8 columns per K step.  V is an MN-major (d contiguous) 128-byte-swizzled tile: 8-key
// groups 1024 bytes apart (stride offset), 64-column slabs of d 16 KB apart (leading
// offset), and a K step of 16 keys advances 2048 bytes.
// F16: P and V in fp16 (FP8 variant) instead of bf16.
template <int D, int K_BEGIN, int K_END, bool F16 = false>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_saddr,
                                         bool accumulate)
{
    constexpr uint32_t idesc = F16 ? ptx::idesc_f32acc(BM, D, 0, 0, 1) : ptx::idesc_bf16_f32(BM, D, 1);
    const uint64_t b0 = ptx::smem_desc_sw128(v_saddr, kChunkBytes, 1024);
#pragma unroll
    for (int k = K_BEGIN; k < K_END; ++k)
        ptx::mma_ts(d_tmem, p_tmem + k * 8, b0 + (uint64_t)(k * 2048 >> 4), idesc, (accumulate || k > 0) ? 1u : 0u);
}

// Pairs of exponentials evaluated on the FMA pipe (exp2_poly2) instead of the MUFU unit:
// every kPolyPeriod-th pair (0 = none).  The MUFU unit (about 4 exp2 per clock per SM
// sub-partition) bounds the softmax; measured on B200 with this kernel, one pair in three
// on the FMA pipe is fastest (one in two runs out of registers, one in four or eight
// leaves the MUFU the bottleneck).
constexpr int kPolyPeriod = 3;

// p = 2^(x * sl2 - m) for NC scores of a row held as raw fp32 bits in x[IN .. IN+NC); the
// p are packed as bf16 pairs into x[OUT .. OUT+NC/2) (OUT <= IN, so every score is read
// before its slot is overwritten) and their fp32 sum is returned.  Lane pairs use packed
// fp32x2 math.
template <int NC, int IN, int OUT, bool F16 = false>
__device__ __forceinline__ float exp2_pack(uint32_t (&x)[128], float sl2, float m)
{
    static_assert(OUT <= IN && NC % 8 == 0, "in-place packing order");
    const float2 c2 = make_float2(sl2, sl2);
    const float2 nm2 = make_float2(-m, -m);
    float2 acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < NC / 2; ++c) {
        const float2 y = __ffma2_rn(make_float2(__uint_as_float(x[IN + 2 * c]), __uint_as_float(x[IN + 2 * c + 1])), c2, nm2);
        float2 e;
        if (kPolyPeriod > 0 && (c + 1) % (kPolyPeriod > 0 ? kPolyPeriod : 1) == 0) {
            e = ptx::exp2_poly2(y);
        } else {
            e.x = ptx::ex2(y.x);
            e.y = ptx::ex2(y.y);
        }
        acc[c & 3] = __fadd2_rn(acc[c & 3], e);
        x[OUT + c] = F16 ? ptx::pack_f16x2(e.x, e.y) : ptx::pack_bf16x2(e.x, e.y);
    }
    const float2 s01 = __fadd2_rn(acc[0], acc[1]);
    const float2 s23 = __fadd2_rn(acc[2], acc[3]);
    const float2 t = __fadd2_rn(s01, s23);
    return t.x + t.y;
}

// Maximum of 64 scores x[IN .. IN+64) (four chains of three-input max).
template <int IN>
__device__ __forceinline__ float row_max64(const uint32_t (&x)[128])
{
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t *v = &x[IN + 16 * i];
        float t = ptx::max3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
        for (int k = 3; k < 15; k += 2) t = ptx::max3(t, __uint_as_float(v[k]), __uint_as_float(v[k + 1]));
        a[i] = fmaxf(t, __uint_as_float(v[15]));
    }
    return fmaxf(ptx::max3(a[0], a[1], a[2]), a[3]);
}

// Set scores of keys past this row's last visible key to -inf (columns [C0, C0+NC)).
template <int C0, int NC>
__device__ __forceinline__ void mask_cols(uint32_t (&x)[128], int kbase, int lim)
{
    if (kbase + C0 + NC - 1 > lim) {
#pragma unroll
        for (int c = C0; c < C0 + NC; ++c)
            if (kbase + c > lim) x[c] = __float_as_uint(-INFINITY);
    }
}

// Set scores of keys before this row's first visible key (sliding window) to -inf.
template <int C0, int NC>
__device__ __forceinline__ void mask_cols_below(uint32_t (&x)[128], int kbase, int first)
{
    if (kbase + C0 < first) {
#pragma unroll
        for (int c = C0; c < C0 + NC; ++c)
            if (kbase + c < first) x[c] = __float_as_uint(-INFINITY);
    }
}

// Four E4M3 bytes b0..b3 -> fp16 pairs (b0, b1) and (b2, b3), exactly (every E4M3 value is
// an fp16 value), by the hardware conversion: measured on B200 in this kernel, about 20%
// faster overall than moving the bit fields with integer operations, which left the two
// widening warps' SM sub-partitions short of issue slots for the softmax warps.
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t x, uint32_t &lo, uint32_t &hi)
{
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(x));
}

// Widen 64 rows (rows 64 cw .. 64 cw + 63) of a 128 x 128 E4M3 V tile (TMA-written, rows of
// 128 bytes, 128-byte swizzle) into the fp16 tile that P V reads: two 64-column slabs, rows
// of 128 bytes, 128-byte swizzle -- the layout of a bf16 V tile.  Lane j of a quarter-warp
// reads chunk j of one row; lanes with chunks 4-7 write their two halves in the other order,
// so every store of a quarter-warp hits eight different bank groups.
__device__ __forceinline__ void widen_v_tile(const uint8_t *src, uint8_t *dst, int cw, int lane)
{
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
        const int idx = i * 32 + lane;
        const int r = 64 * cw + (idx >> 3);
        const int c = idx & 7;  // dims 16c .. 16c + 15
        const uint4 x = *reinterpret_cast<const uint4 *>(src + r * 128 + ((c ^ (r & 7)) << 4));
        uint4 a, b;  // dims 16c .. +7 and 16c + 8 .. +15 as fp16
        e4m3x4_to_f16(x.x, a.x, a.y);
        e4m3x4_to_f16(x.y, a.z, a.w);
        e4m3x4_to_f16(x.z, b.x, b.y);
        e4m3x4_to_f16(x.w, b.z, b.w);
        uint8_t *row = dst + (c >> 2) * kChunkBytes + r * 128;
        const int k0 = 2 * (c & 3);
        uint4 *pa = reinterpret_cast<uint4 *>(row + ((k0 ^ (r & 7)) << 4));
        uint4 *pb = reinterpret_cast<uint4 *>(row + (((k0 + 1) ^ (r & 7)) << 4));
        if (c < 4) {
            *pa = a;
            *pb = b;
        } else {
            *pb = b;
            *pa = a;
        }
    }
}

// A wait that ignores the stop flag, used only to let copies and MMAs already in
// flight finish before the CTA leaves.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (ptx::mbar_test(bar, parity)) return;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_test(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > limit_ns) {
            raise_error(kErrTimeout);
            return;
        }
    }
}

}  // namespace prefill

// SPLIT_P: hand P to the MMA warp in two halves (used for head-pair units; measured to
// help the grouped-query tiling and to cost a little on the row-pair tiling).  FP8: Q, K
// and V in E4M3 (d = 128 only).
template <int D, bool OUT_F32, bool SPLIT_P, bool WINDOW, bool FP8 = false>
__global__ void __launch_bounds__(prefill::kThreads, 1)
    fa_prefill_kernel(const __grid_constant__ PrefillParams p)
{
    using namespace prefill;
    using C = Cfg<D, FP8>;
    static_assert(!FP8 || D == 128, "FP8 prefill: head dim 128");
    constexpr int kBoxes = FP8 ? 1 : D / 64;  // 128-byte column boxes per loaded tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *kv_full = bars;
    uint64_t *kv_empty = bars + C::kStages;
    uint64_t *q_full = bars + 2 * C::kStages;  // [set * 2 + tile]
    uint64_t *q_empty = q_full + 4;             // [set * 2 + tile]
    uint64_t *s_full = q_full + 8;
    uint64_t *p_ready = q_full + 10;
    uint64_t *o_done = q_full + 12;
    uint64_t *o_free = q_full + 14;
    uint64_t *teardown = q_full + 16;
    uint64_t *p_half = q_full + 17;     // [2]: first 64 keys of P_s written
    uint64_t *v16_full = q_full + 19;   // FP8 [2]: widened V tile written (one arrive per widening warp)
    uint64_t *v16_empty = q_full + 21;  // FP8 [2]: widened V tile read by its last P V
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::kMiscOff);
    int *stop_flag = reinterpret_cast<int *>(smem + C::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            ptx::mbar_init(&kv_full[i], 1);
            // FP8: the V stages (odd) are released by the two widening warps
            ptx::mbar_init(&kv_empty[i], (FP8 && (i & 1)) ? 2 : 1);
        }
        if (FP8) {
            for (int i = 0; i < 2; ++i) {
                ptx::mbar_init(&v16_full[i], 2);
                ptx::mbar_init(&v16_empty[i], 1);
            }
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&q_full[s], 1);
            ptx::mbar_init(&q_full[2 + s], 1);
            // a Q slot is free again once its last S MMA is done (MMA commit) and the
            // epilogue, which stages O through the same slot, has stored it (one arrive
            // per warp of the softmax warpgroup)
            ptx::mbar_init(&q_empty[s], 5);
            ptx::mbar_init(&q_empty[2 + s], 5);
            ptx::mbar_init(&s_full[s], 1);
            ptx::mbar_init(&p_ready[s], 128);
            ptx::mbar_init(&p_half[s], 128);
            ptx::mbar_init(&o_done[s], 1);
            ptx::mbar_init(&o_free[s], 128);
        }
        ptx::mbar_init(teardown, 1);
        *stop_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 9) {
        ptx::tmem_alloc(tmem_holder, 512);
        ptx::tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        ptx::tma_prefetch_desc(&p.tm_q);
        ptx::tma_prefetch_desc(&p.tm_k);
        ptx::tma_prefetch_desc(&p.tm_v);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const StopFlag sf{stop_flag, p.wait_limit_ns};

    const uint32_t q_saddr0 = ptx::smem_addr(smem + C::kQOff);
    const uint32_t kv_saddr0 = ptx::smem_addr(smem + C::kKVOff);
    const uint32_t v16_saddr0 = ptx::smem_addr(smem + C::kV16Off);

    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp runs the loop (every value is warp-uniform); one elected lane
        // issues the copies.
        ptx::regs_decrease<kRegsLow>();
        const bool leader = ptx::elect_one();
        uint32_t kv_it = 0;
        uint32_t q_fills[4] = {0u, 0u, 0u, 0u};
        bool ok = true;
        // Q tiles of unit number i (in this CTA's order) go to Q set i & 1 and are loaded one
        // unit ahead.  The slot of unit i + 1 is released only by unit i - 1's epilogue, so
        // those loads are issued whenever the slot is free, between K/V loads, without ever
        // holding up the K/V stream; only at the end of a unit does the warp block on them.
        auto issue_q = [&](const Unit &uw, uint32_t i, int s) {
            const int qi = 2 * (int)(i & 1u) + s;
            ++q_fills[qi];
            if (leader) {
                ptx::mbar_arrive_expect_tx(&q_full[qi], C::kInTileBytes);
                const int h = s ? uw.h1 : uw.h0;
                const int r = s ? uw.r1 : uw.r0;
                uint8_t *dst = smem + C::kQOff + qi * C::kInTileBytes;
#pragma unroll
                for (int c = 0; c < kBoxes; ++c)
                    ptx::tma_load_4d(dst + c * kChunkBytes, &p.tm_q, &q_full[qi], 64 * c, r, h, uw.b);
            }
            __syncwarp();
        };
        auto q_slot = [&](uint32_t i, int s) { return &q_empty[2 * (int)(i & 1u) + s]; };
        auto q_free_parity = [&](uint32_t i) { return ((i >> 1) & 1u) ^ 1u; };
        Unit w, wn;
        int u = next_unit<WINDOW>(p, 2 * (int)blockIdx.x, w);
        uint32_t i = 0;
        for (int s = 0; ok && u >= 0 && s < 2; ++s) {
            if (!wait_warp(q_slot(0, s), q_free_parity(0), sf)) ok = false;
            else issue_q(w, 0, s);
        }
        for (; ok && u >= 0; ++i) {
            const int un = next_unit<WINDOW>(p, unit_step(u), wn);
            int q_next = (un >= 0) ? 0 : 2;  // look-ahead Q tiles already issued
            for (int j = w.a0; j < w.n1 && ok; ++j) {
                for (int kv = 0; kv < 2; ++kv) {
                    const uint32_t st = kv_it % C::kStages;
                    const uint32_t ph = (kv_it / C::kStages) & 1u;
                    if (!wait_warp(&kv_empty[st], ph ^ 1u, sf)) { ok = false; break; }
                    if (leader) {
                        ptx::mbar_arrive_expect_tx(&kv_full[st], C::kInTileBytes);
                        uint8_t *dst = smem + C::kKVOff + st * C::kInTileBytes;
                        const CUtensorMap *map = kv ? &p.tm_v : &p.tm_k;
#pragma unroll
                        for (int c = 0; c < kBoxes; ++c)
                            ptx::tma_load_4d(dst + c * kChunkBytes, map, &kv_full[st], 64 * c, BN * j, w.g, w.b);
                    }
                    __syncwarp();
                    ++kv_it;
                    while (q_next < 2 &&
                           __all_sync(0xffffffffu, ptx::mbar_test(q_slot(i + 1, q_next), q_free_parity(i + 1)))) {
                        issue_q(wn, i + 1, q_next);
                        ++q_next;
                    }
                }
            }
            for (; ok && q_next < 2; ++q_next) {
                if (!wait_warp(q_slot(i + 1, q_next), q_free_parity(i + 1), sf)) ok = false;
                else issue_q(wn, i + 1, q_next);
            }
            u = un;
            w = wn;
        }
        // Let every copy this warp started land before the CTA can exit.
        if (leader) {
            for (uint32_t st = 0; st < (uint32_t)C::kStages && st < kv_it; ++st) {
                const uint32_t last = kv_it - 1 - ((kv_it - 1 - st) % C::kStages);
                drain_wait(&kv_full[st], (last / C::kStages) & 1u, p.wait_limit_ns);
            }
            for (int qi = 0; qi < 4; ++qi)
                if (q_fills[qi] > 0) drain_wait(&q_full[qi], (q_fills[qi] - 1) & 1u, p.wait_limit_ns);
        }
        __syncwarp();
    } else if (warp == 9) {
        // --------------------------------------------------------------- MMA issuer
        // The whole warp runs the loop, so descriptors and addresses are warp-uniform;
        // one elected lane issues each group of MMAs and its commits.
        ptx::regs_decrease<kRegsLow>();
        const bool leader = ptx::elect_one();
        const bool signal_s = !p.selftest_no_s_signal;
        uint32_t kv_it = 0, units = 0;
        uint32_t p_ph[2] = {0u, 0u};
        bool ok = true;
        // The P V of tile 1's last key tile is not issued at the end of its unit but carried
        // into the next unit's first iteration, after that unit's first S0 MMA: the
        // S0 / PV1 / S1 / PV0 ping-pong then runs on across unit boundaries instead of
        // draining the tensor pipe at every unit.
        bool pend = false, pend_acc = false, pend_free = false;
        uint32_t pend_v = 0, pend_free_par = 0;
        // P V of Q tile s.  With SPLIT_P in two halves: keys 0-63 as soon as the softmax
        // has written that half of P, keys 64-127 when the whole tile is done.
        auto issue_pv_halves = [&](int s, uint32_t v_stage, bool acc, bool need_free, uint32_t fpar) -> bool {
            const uint32_t d_tmem = tmem + 256 + 128 * s, p_tmem = tmem + 128 * s;
            // v_stage: the K/V ring stage of V, or (FP8) the widened V tile
            const uint32_t v_saddr = (FP8 ? v16_saddr0 : kv_saddr0) + v_stage * C::kTileBytes;
            if (SPLIT_P) {
                if (need_free && !wait_warp(&o_free[s], fpar, sf)) return false;
                if (!wait_warp(&p_half[s], p_ph[s], sf)) return false;
                ptx::tc_fence_after();
                if (leader) issue_pv<D, 0, 4, FP8>(d_tmem, p_tmem, v_saddr, acc);
                __syncwarp();
                if (!wait_warp(&p_ready[s], p_ph[s], sf)) return false;
                p_ph[s] ^= 1u;
                ptx::tc_fence_after();
                if (leader) issue_pv<D, 4, 8, FP8>(d_tmem, p_tmem, v_saddr, true);
            } else {
                if (!wait_warp(&p_ready[s], p_ph[s], sf)) return false;
                p_ph[s] ^= 1u;
                if (need_free && !wait_warp(&o_free[s], fpar, sf)) return false;
                ptx::tc_fence_after();
                if (leader) issue_pv<D, 0, 8, FP8>(d_tmem, p_tmem, v_saddr, acc);
            }
            __syncwarp();
            return true;
        };
        auto issue_pv1 = [&](uint32_t v_stage, bool acc, bool need_free, uint32_t fpar, bool last) -> bool {
            if (!issue_pv_halves(1, v_stage, acc, need_free, fpar)) return false;
            if (leader) {
                ptx::mma_commit(FP8 ? &v16_empty[v_stage] : &kv_empty[v_stage]);
                if (last) ptx::mma_commit(&o_done[1]);
            }
            __syncwarp();
            return true;
        };
        Unit w;
        for (int u = next_unit<WINDOW>(p, 2 * (int)blockIdx.x, w); ok && u >= 0; u = next_unit<WINDOW>(p, unit_step(u), w)) {
            const uint32_t free_par = (units & 1u) ^ 1u;  // first unit passes at once
            const uint32_t qset = units & 1u;
            const uint32_t q_par = (units >> 1) & 1u;
            uint64_t *qf = q_full + 2 * qset;
            uint64_t *qe = q_empty + 2 * qset;
            const uint32_t q_saddr = q_saddr0 + 2 * qset * C::kInTileBytes;
            if (!wait_warp(&qf[0], q_par, sf) || !wait_warp(&qf[1], q_par, sf)) break;
            ptx::tc_fence_after();
            uint32_t prev_v = 0;
            // Key tile j feeds S0 / P V0 when a0 <= j < n0 and S1 / P V1 when a1 <= j < n1.
            for (int j = w.a0; j < w.n1; ++j) {
                const uint32_t ks = kv_it % C::kStages;
                const uint32_t kph = (kv_it / C::kStages) & 1u;
                // V of this key tile: its ring stage, or (FP8) its widened tile (alternating)
                const uint32_t vs = FP8 ? (kv_it >> 1) & 1u : (kv_it + 1) % C::kStages;
                const uint32_t vph = FP8 ? (kv_it >> 2) & 1u : ((kv_it + 1) / C::kStages) & 1u;
                uint64_t *v_ready = FP8 ? &v16_full[vs] : &kv_full[vs];
                uint64_t *v_release = FP8 ? &v16_empty[vs] : &kv_empty[vs];
                if (!wait_warp(&kv_full[ks], kph, sf)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t k_saddr = kv_saddr0 + ks * C::kInTileBytes;
                if (j < w.n0) {
                    if (leader) {
                        if (FP8) issue_qk_fp8(tmem + 0, q_saddr, k_saddr);
                        else issue_qk<D>(tmem + 0, q_saddr, k_saddr);
                        if (signal_s) ptx::mma_commit(&s_full[0]);
                        if (j == w.n0 - 1) ptx::mma_commit(&qe[0]);
                    }
                    __syncwarp();
                }
                if (j > w.a1) {
                    if (!issue_pv1(prev_v, j - 1 > w.a1, j - 1 == w.a1, free_par, false)) { ok = false; break; }
                } else if (pend) {
                    if (!issue_pv1(pend_v, pend_acc, pend_free, pend_free_par, true)) { ok = false; break; }
                    pend = false;
                }
                if (leader) {
                    if (j >= w.a1) {
                        if (FP8) issue_qk_fp8(tmem + 128, q_saddr + C::kInTileBytes, k_saddr);
                        else issue_qk<D>(tmem + 128, q_saddr + C::kInTileBytes, k_saddr);
                        if (signal_s) ptx::mma_commit(&s_full[1]);
                    }
                    ptx::mma_commit(&kv_empty[ks]);
                    if (j == w.n1 - 1) ptx::mma_commit(&qe[1]);
                }
                __syncwarp();
                if (!wait_warp(v_ready, vph, sf)) { ok = false; break; }
                if (j < w.n0) {
                    if (!issue_pv_halves(0, vs, j > w.a0, j == w.a0, free_par)) { ok = false; break; }
                    if (leader && j == w.n0 - 1) ptx::mma_commit(&o_done[0]);
                    __syncwarp();
                }
                // a V tile that Q tile 1 never reads is released here (sliding window)
                if (j < w.a1) {
                    if (leader) ptx::mma_commit(v_release);
                    __syncwarp();
                }
                prev_v = vs;
                kv_it += 2;
            }
            if (!ok) break;
            pend = true;
            pend_v = prev_v;
            pend_acc = w.n1 - 1 > w.a1;
            pend_free = w.n1 - 1 == w.a1;
            pend_free_par = free_par;
            ++units;
        }
        if (ok && pend) issue_pv1(pend_v, pend_acc, pend_free, pend_free_par, true);
        // Every MMA and commit issued above completes before the CTA can exit.
        if (leader) {
            ptx::mma_commit(teardown);
            drain_wait(teardown, 0, p.wait_limit_ns);
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax warps
        ptx::regs_increase<kRegsHigh>();
        const int s = warp >> 2;              // which Q tile of the unit
        const int tid = threadIdx.x & 127;    // row inside the tile = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + 128u * s;        // S_s, and P_s over it
        const uint32_t tO = tmem + lane_base + 256u + 128u * s;  // O_s
        float sl2 = p.scale_log2;
        uint32_t s_ph = 0, units = 0;
        Unit w;
        for (int u = next_unit<WINDOW>(p, 2 * (int)blockIdx.x, w); u >= 0; u = next_unit<WINDOW>(p, unit_step(u), w)) {
            const int h = s ? w.h1 : w.h0;
            const int r0 = s ? w.r1 : w.r0;
            const int a = s ? w.a1 : w.a0;
            const int n = s ? w.n1 : w.n0;
            const int row = r0 + tid;
            const int lim = p.causal ? min(row + (p.Nk - p.Nq), p.Nk - 1) : p.Nk - 1;
            const int first = WINDOW ? row + (p.Nk - p.Nq) - p.window + 1 : 0;
            // FP8: the scores are products of E4M3 codes; the head scales join the softmax scale
            if (FP8) {
                const bool okq = in_bounds(h, p.Hq), okk = in_bounds(w.g, p.Hkv);
                sl2 = p.scale_log2 * (okq ? p.q_scale[h] : 1.f) * (okk ? p.k_scale[w.g] : 1.f);
            }
            // l: sum of the fp32 weights (gives the LSE).  lo: normaliser of O, the same sum
            // corrected, tile by tile, by the bf16 rounding of the tile's largest weight --
            // the rounding the P V product actually saw.  For a row dominated by one key
            // this makes O exactly that key's value row, as it should be.
            float m = -INFINITY, l = 0.f, lo = 0.f;
            bool ok = true;
            for (int j = a; j < n; ++j) {
                if (!wait_warp(&s_full[s], s_ph, sf)) { ok = false; break; }
                s_ph ^= 1u;
                ptx::tc_fence_after();
                uint32_t x[128];
                const int kbase = BN * j;
                float alpha = 1.f, sum, mx;
                bool rescale = false;
                // Scores of this tile, masked past the row's last visible key; the tile
                // maximum; lazy update of the reference maximum m (moved only when the new
                // one exceeds it by more than kLazyThreshold, which then rescales O).
                ptx::tmem_ld32(tS + 0, &x[0]);
                ptx::tmem_ld32(tS + 32, &x[32]);
                ptx::tmem_ld32(tS + 64, &x[64]);
                ptx::tmem_ld32(tS + 96, &x[96]);
                ptx::tmem_wait_ld();
                mask_cols<0, 128>(x, kbase, lim);
                if (WINDOW) mask_cols_below<0, 128>(x, kbase, first);
                mx = fmaxf(row_max64<0>(x), row_max64<64>(x)) * sl2;
                if (j == a) {
                    m = mx;  // O is not written yet: the first P V overwrites it
                } else if (mx - m > (FP8 ? kLazyThresholdF16 : kLazyThreshold)) {
                    // (also taken when m is still -inf: the row's window had not started)
                    alpha = ptx::ex2(m - mx);
                    m = mx;
                    rescale = true;
                }
                // reference maximum for the exponentials: with a window, 0 while the row
                // has seen no key, so that masked scores give exactly 0 instead of
                // -inf - (-inf).  (Without one, every row sees a key in its first tile.)
                const float mref = (WINDOW && m == -INFINITY) ? 0.f : m;
                // Rare (lazy) rescale of the partial output, before any P V of this tile is
                // issued (P V of the previous tile is complete: the commit that signalled
                // this S tile covers it); warp-uniform because TMEM accesses are collective.
                auto rescale_o = [&]() {
                    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t ov[32];
                            ptx::tmem_ld32(tO + 32 * c, ov);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                            ptx::tmem_st32(tO + 32 * c, ov);
                        }
                    }
                };
                if (SPLIT_P) {
                    // the first 64 keys of P are handed to the MMA warp while the second
                    // half is still being computed
                    rescale_o();
                    sum = exp2_pack<64, 0, 0, FP8>(x, sl2, mref);
                    ptx::tmem_st32(tS + 0, &x[0]);
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(&p_half[s]);
                    sum += exp2_pack<64, 64, 32, FP8>(x, sl2, mref);
                    ptx::tmem_st32(tS + 32, &x[32]);
                } else {
                    sum = exp2_pack<64, 0, 0, FP8>(x, sl2, mref) + exp2_pack<64, 64, 32, FP8>(x, sl2, mref);
                    ptx::tmem_st32(tS + 0, &x[0]);
                    ptx::tmem_st32(tS + 32, &x[32]);
                    rescale_o();
                }
                ptx::tmem_wait_st();
                const float p_top = ptx::ex2(mx - mref);  // the tile's largest weight (0 if masked)
                const float p_top_bf = FP8 ? __half2float(__float2half_rn(p_top))
                                           : __uint_as_float(ptx::pack_bf16x2(p_top, 0.f) << 16);
                l = l * alpha + sum;
                lo = lo * alpha + sum + (p_top_bf - p_top);
                ptx::tc_fence_before();
                ptx::mbar_arrive(&p_ready[s]);
            }
            if (!ok) break;
            // ------------------------------------------------------------- epilogue
            // O_s / lo leaves TMEM as soon as it is read (o_free lets the next unit's first
            // P V overwrite it).  bf16 output is staged, 128-byte swizzled, in this unit's Q
            // slot -- no MMA reads it any more -- and each warp writes its own 32 rows with
            // one TMA store, then hands its part of the slot back to the producer, so no
            // warp waits for another.  fp32 output is stored row by row.
            if (!wait_warp(&o_done[s], units & 1u, sf)) break;
            ptx::tc_fence_after();
            const bool valid = row < p.Nq;
            // FP8: the widened V holds the E4M3 codes; v_scale restores V
            const float inv_l = FP8 ? (in_bounds(w.g, p.Hkv) ? p.v_scale[w.g] : 1.f) / lo : 1.f / lo;
            long long orow = ((long long)w.b * p.Hq + h) * (long long)p.Nq + (valid ? row : 0);  // LSE index
            if (kDebugChecks) orow += p.debug_lse_offset;
            const int qi = 2 * (int)(units & 1u) + s;
            uint32_t ov[D];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) ptx::tmem_ld32(tO + 32 * c, &ov[32 * c]);
            ptx::tmem_wait_ld();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&o_free[s]);
            if (OUT_F32) {
                const long long ooff = w.b * p.o_sb + h * p.o_sh + (long long)row * p.o_sn;
                if (valid && in_bounds(ooff + D - 1, (long long)p.B * p.Hq * p.Nq * D)) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + ooff);
#pragma unroll
                    for (int e = 0; e < D / 4; ++e)
                        dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv_l,
                                             __uint_as_float(ov[4 * e + 1]) * inv_l,
                                             __uint_as_float(ov[4 * e + 2]) * inv_l,
                                             __uint_as_float(ov[4 * e + 3]) * inv_l);
                }
                if (lane == 0) ptx::mbar_arrive(&q_empty[qi]);
            } else if (FP8) {
                // The E4M3 Q slot (16 KB) holds one 64-column slab of the bf16 O tile: two
                // rounds, each warp staging and storing its own 32 rows.
                uint8_t *stage = smem + C::kQOff + qi * C::kInTileBytes;
                const int wr = 32 * (warp & 3);  // this warp's rows of the tile
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t *src = &ov[64 * c + 8 * e];
                        uint4 v4;
                        v4.x = ptx::pack_bf16x2(__uint_as_float(src[0]) * inv_l, __uint_as_float(src[1]) * inv_l);
                        v4.y = ptx::pack_bf16x2(__uint_as_float(src[2]) * inv_l, __uint_as_float(src[3]) * inv_l);
                        v4.z = ptx::pack_bf16x2(__uint_as_float(src[4]) * inv_l, __uint_as_float(src[5]) * inv_l);
                        v4.w = ptx::pack_bf16x2(__uint_as_float(src[6]) * inv_l, __uint_as_float(src[7]) * inv_l);
                        *reinterpret_cast<uint4 *>(stage + tid * 128 + ((e ^ (tid & 7)) << 4)) = v4;
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && r0 + wr < p.Nq && in_bounds(h, p.Hq) && in_bounds(w.b, p.B)) {  // (rows past Nq are never stored)
                        ptx::tma_store_4d(&p.tm_o, stage + wr * 128, 64 * c, r0 + wr, h, w.b);
                        ptx::bulk_commit_group();
                        ptx::bulk_wait_group_read0();  // the slab's rows are restaged next round
                    }
                    __syncwarp();
                }
                if (lane == 0) ptx::mbar_arrive(&q_empty[qi]);
            } else {
                uint8_t *stage = smem + C::kQOff + qi * C::kTileBytes;
#pragma unroll
                for (int e = 0; e < D / 8; ++e) {
                    uint4 v4;
                    v4.x = ptx::pack_bf16x2(__uint_as_float(ov[8 * e + 0]) * inv_l, __uint_as_float(ov[8 * e + 1]) * inv_l);
                    v4.y = ptx::pack_bf16x2(__uint_as_float(ov[8 * e + 2]) * inv_l, __uint_as_float(ov[8 * e + 3]) * inv_l);
                    v4.z = ptx::pack_bf16x2(__uint_as_float(ov[8 * e + 4]) * inv_l, __uint_as_float(ov[8 * e + 5]) * inv_l);
                    v4.w = ptx::pack_bf16x2(__uint_as_float(ov[8 * e + 6]) * inv_l, __uint_as_float(ov[8 * e + 7]) * inv_l);
                    // 16-byte chunk e of the row: slab e / 8, chunk (e % 8) swizzled by row % 8
                    const int slab = e >> 3, chunk = (e & 7) ^ (tid & 7);
                    *reinterpret_cast<uint4 *>(stage + slab * kChunkBytes + tid * 128 + chunk * 16) = v4;
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int wr = 32 * (warp & 3);  // this warp's rows of the tile
                    if (r0 + wr < p.Nq && in_bounds(h, p.Hq) && in_bounds(w.b, p.B)) {  // (rows past Nq are never stored)
#pragma unroll
                        for (int c = 0; c < D / 64; ++c)
                            ptx::tma_store_4d(&p.tm_o, stage + c * kChunkBytes + wr * 128, 64 * c, r0 + wr, h, w.b);
                        ptx::bulk_commit_group();
                        ptx::bulk_wait_group_read0();
                    }
                    ptx::mbar_arrive(&q_empty[qi]);
                }
            }
            if (valid && in_bounds(orow, (long long)p.B * p.Hq * p.Nq)) p.lse[orow] = (m + ptx::lg2(l)) * kLn2;
            ++units;
        }
        if (!OUT_F32 && lane == 0) ptx::bulk_wait_group0();  // stores complete before exit
    }

    else {
        ptx::regs_decrease<kRegsLow>();
        if (FP8) {
            // -------------------------------------------------------- V widening (FP8)
            // Warps 10 and 11 follow the producer's key-tile order and turn each E4M3 V
            // tile (odd ring stage) into the fp16 tile P V reads, rows 64 (warp - 10) on.
            const int cw = warp - 10;
            uint32_t kv_it = 0;
            bool ok = true;
            Unit w;
            for (int u = next_unit<WINDOW>(p, 2 * (int)blockIdx.x, w); ok && u >= 0;
                 u = next_unit<WINDOW>(p, unit_step(u), w)) {
                for (int j = w.a0; j < w.n1; ++j, kv_it += 2) {
                    const uint32_t st = (kv_it + 1) % C::kStages;
                    const uint32_t ph = ((kv_it + 1) / C::kStages) & 1u;
                    const uint32_t vb = (kv_it >> 1) & 1u;
                    const uint32_t vpar = (kv_it >> 2) & 1u;
                    if (!wait_warp(&kv_full[st], ph, sf) || !wait_warp(&v16_empty[vb], vpar ^ 1u, sf)) {
                        ok = false;
                        break;
                    }
                    widen_v_tile(smem + C::kKVOff + st * C::kInTileBytes, smem + C::kV16Off + vb * C::kTileBytes,
                                 cw, lane);
                    ptx::fence_proxy_async_smem();  // the tensor core reads these through the async proxy
                    __syncwarp();
                    if (lane == 0) {
                        ptx::mbar_arrive(&v16_full[vb]);
                        ptx::mbar_arrive(&kv_empty[st]);
                    }
                }
            }
        }
    }
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

}  // namespace fa
