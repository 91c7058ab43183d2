// fa_decode_sm100.cuh -- split-KV decode over a KV cache, with a log-sum-exp merge.
//
// Decode (one new query row per sequence) reads the whole cache every step and does
// only 4 flops per byte, so it is bound by HBM bandwidth (youngju.dev "attention
// variants", section 7).  The cache of one (sequence, key/value head) is contiguous, so
// it is cut into chunks of kChunk keys; a work item is one chunk for the RG query heads of
// one key/value head group.
//
// Only valid items are enumerated, so every CTA (bf16) or worker warp (FP8) gets the same
// number to within one.  Both split kernels are persistent, 3 CTAs per SM, one producer
// warp streaming blocks of cache rows into shared memory with TMA and four consumer warps
// running mma.sync with the query heads in N = 8 and keys (S^T = K Q^T) or head dims
// (O^T = V^T P^T) in M = 16, so no MMA row is padding:
//   bf16 split kernel: the four consumer warps share one ring of 64-row stages and work on
//     one item together: K pass (each warp 16 keys of every stage, scores to shared
//     memory), chunk softmax (max, p = 2^(s - max), sum), V pass (each warp a quarter of
//     the head dims over all keys), then the normalised partial and its log2-sum-exp.
//   FP8 split kernel: every consumer warp is an independent worker with items of its own
//     and a two-slot ring (the item's K and V blocks of 64 keys, 8 KB each) that the
//     producer refills as soon as the worker frees a slot, polling the four rings in turn.
//     Per block a worker computes S^T, runs the online softmax of youngju.dev section 3 on
//     it in registers (running max and sum per head; the output is rescaled when the max
//     grows), passes P through a small shared-memory tile of its own (to put the heads in
//     N again) and accumulates O^T; no warp ever waits for another.  (Measured on B200:
//     this arrangement is the faster one for FP8, whose blocks need more arithmetic per
//     byte; for bf16 the shared-ring arrangement is.)
//   merge kernel, one CTA per (head, sequence): M = max of the partial log-sum-exps,
//     w_s = 2^(lse_s - M), o = sum_s w_s o_s / sum_s w_s, lse = M + log2 sum_s w_s.
// The merge is the same rescaling the online softmax applies between key blocks
// (youngju.dev section 3), applied across chunks.
//
// Paged caches (youngju.dev section 5: the cache cut into fixed-size blocks managed like
// virtual-memory pages) change only the producer's addressing: the tensor maps span the
// page pool (num_pages * Hkv planes of page_size rows), the producer looks up the physical
// pages of an item's keys in the block table (one entry per lane) and copies boxes of
// box_rows rows, a power of two that divides page_size, so no box straddles two pages.
//
// FP8 caches (E4M3 bytes with one dequantization scale per K/V head for K and one for V;
// youngju.dev sections 5 and 7 name FP8 KV caches) halve the bytes read.  Each pair of E4M3
// values becomes a pair of fp16 values in registers by the hardware conversion
// (cvt.rn.f16x2.e4m3x2 of 16 bits, exact: every E4M3 value is an fp16 value), and the same
// mma.sync tiles run on fp16 operands:
//   K: ldmatrix (not transposed) hands a lane 4 consecutive dims of one key; the two 16-bit
//     halves of that register, dims (0, 1) and (2, 3), convert directly into the lane's A
//     registers of the MMA's contraction index 2tig + {0, 1} and 2tig + {8, 9}, and q is
//     loaded in the same order (so no byte moves are needed).  q is scaled per row by an
//     exact power of two 2^e so that its largest element lies in [2^14, 2^15) before the
//     fp16 conversion (every bf16 value in that range is an fp16 value); k_scale * 2^-e is
//     applied to the fp32 scores.
//   V: a transposing 16-bit ldmatrix hands a lane 2 dims x 2 keys as bytes
//     {key 0 dim 0, key 0 dim 1, key 1 dim 0, key 1 dim 1}: bytes (0, 2) are the key pair
//     of the even dim and (1, 3) that of the odd dim, the A rows of the even and the odd
//     output dims; one byte permute per register puts them in the order (0, 2, 1, 3) so
//     that its two halves convert directly.  P is converted to fp16 and v_scale is applied
//     with the final 1 / l.
// (Measured on B200: the hardware conversion for K and V is 7% faster on the FP8 decode
// workload than moving the E4M3 bit fields into fp16 with integer operations, whose
// arithmetic kept the ALU pipe the busiest unit of the kernel.)
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "fa_common.cuh"
#include "ptx_sm100.cuh"

namespace fa {

struct DecodeParams {
    CUtensorMap tm_k;         // kcache as (D, Nmax, B*Hkv) bf16, box (64, 64, 1), 128B swizzle;
                              // paged: kpages as (D, page_size, num_pages*Hkv), box (64, box_rows, 1)
    CUtensorMap tm_v;         // vcache / vpages, same shape
    const __nv_bfloat16 *q;   // (B, Hq, D)
    const int *seqlens;       // (B)
    float *part_o;            // (B, Hq, S_max, D)  normalised partial outputs
    float *part_lse;          // (B, Hq, S_max)     partial log2-sum-exp (scaled scores)
    __nv_bfloat16 *o;         // (B, Hq, D) bf16 output, or
    float *o_f32;             // (B, Hq, D) fp32 output when not null (o is then unused)
    float *lse;               // (B, Hq) natural log, may be null
    int B, Hq, Hkv, Nmax, R, S_max;
    int n_hg;      // head groups: Hq / RG
    int n_items;   // S_max * B * n_hg: an upper bound on the work items (sizes the grid)
    float scale_log2;
    unsigned long long wait_limit_ns;
    // FP8 cache only: per K/V head dequantization scales (Hkv each)
    const float *k_scale, *v_scale;
    // paged cache only (Nmax = page_size * max_pages)
    const int *block_table;   // (B, max_pages) physical page of each logical page
    int page_size, max_pages, num_pages;
    int box_rows;             // rows per copy: a power of two <= 64 that divides page_size
    // time-limit self-test: the producer of every CTA withholds its first copy (neither the
    // arrive nor the copy is issued), so the consumers' first wait must run out
    int selftest_no_full;
};

namespace decode {

constexpr int kChunk = 256;        // keys per work item
constexpr int kWarps = 4;          // consumer warps
constexpr int kThreads = 32 * (kWarps + 1);
constexpr int kCtasPerSm = 3;
constexpr float kLn2 = 0.6931471805599453f;

// bf16 kernel: a ring of stages of kSub key rows shared by the four consumer warps.
constexpr int kSub = 64;               // key rows per ring stage
constexpr int kBoxBytes = kSub * 128;  // one 128-byte column box of a stage

template <int D, int RG>
struct SplitCfg {
    static constexpr int kRowChunks = D * 2 / 16;                      // 16-byte chunks per row
    static constexpr int kStageBytes = (D / 64) * kBoxBytes;
    static constexpr int kStages = (D == 128) ? 4 : 8;                 // 64 KB ring
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kScoreOff = kRingBytes;                       // float [RG][kChunk]
    static constexpr int kMOff = kScoreOff + RG * kChunk * 4;          // float m[RG], l[RG]
    static constexpr int kBarOff = (kMOff + 2 * RG * 4 + 15) & ~15;    // full[S], empty[S], group
    static constexpr int kStopOff = kBarOff + (2 * kStages + 1) * 8;
    static constexpr int kSmemBytes = kStopOff + 16 + 1024;            // + alignment slack
};

// FP8 kernel: every consumer warp owns a two-slot ring of 8 KB blocks (64 keys of 128 E4M3
// bytes), one K block and one V block.
constexpr int kStageBytes = 8192;
constexpr int kSK = 64;                // keys per block

template <int RG>
struct WorkerCfg {
    static constexpr int kPStride = kSK + 8;                             // fp16 P row (padded)
    static constexpr int kPOff = kWarps * 2 * kStageBytes;               // after the rings [warp][K, V]
    static constexpr int kPBytes = 8 * kPStride * 2;                     // [8 heads][kPStride]
    static constexpr int kBarOff = (kPOff + kWarps * kPBytes + 15) & ~15;  // full[warp][2], empty[warp][2]
    static constexpr int kStopOff = kBarOff + kWarps * 4 * 8;
    static constexpr int kSmemBytes = kStopOff + 16 + 1024;              // + alignment slack
};

__device__ __forceinline__ int clamp_len(int L, int Nmax)
{
    return L < 0 ? 0 : (L > Nmax ? Nmax : L);
}

// Byte offset of 16-byte chunk `c` of row `r` of a block written by TMA with 128-byte
// swizzle: column boxes of BOX bytes (rows of 128 bytes), the chunk index within the box
// XORed with the row's index modulo 8.
template <int BOX = kBoxBytes>
__device__ __forceinline__ uint32_t stage_offset(int r, int c)
{
    return (uint32_t)((c >> 3) * BOX + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) { return ptx::pack_bf16x2(lo, hi); }

// E4M3 bytes (0, 1) and (2, 3) of x to two packed fp16 pairs (low byte to the low half), exactly
__device__ __forceinline__ void e4m3_halves_f16x2(uint32_t x, uint32_t &lo, uint32_t &hi)
{
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(x));
}

}  // namespace decode

// Work items.  Only the valid items are enumerated -- (sequence b, chunk c < ceil(L_b /
// kChunk), head group hg), sequence-major -- and item v goes to worker v mod (number of
// workers: CTAs for bf16, consumer warps for FP8), so every worker gets the same number of
// items to within one whatever the lengths.  Inside a sequence the order is a layout
// choice: HEAD_MAJOR (head group, then chunk) makes the items running at one time read
// neighbouring chunks of one head, which suits the contiguous bf16 cache (+1.9% measured
// on B200 against chunk-major); chunk-major (chunk, then head group) makes them read the
// heads of one page, which suits the paged pool, and measured 2.3% faster for the FP8
// worker kernel.  The item -> (b, chunk)
// map needs the prefix sums of the chunk counts; each warp that walks the items keeps a
// cursor on the sequence of its current item and moves it forward 32 sequences per step (a
// warp scan of their chunk counts).  Every call below is made by all 32 lanes of a warp with
// warp-uniform arguments.
__device__ __forceinline__ int seq_chunks(const DecodeParams &p, int b)
{
    return (decode::clamp_len(p.seqlens[b], p.Nmax) + decode::kChunk - 1) / decode::kChunk;
}

// Number of valid items of the launch.
__device__ __forceinline__ int count_items(const DecodeParams &p)
{
    const int lane = threadIdx.x & 31;
    int s = 0;
    for (int b = lane; b < p.B; b += 32) s += seq_chunks(p, b);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s * p.n_hg;
}

struct ItemCursor {
    int b = -1;    // sequence of the last item found
    int base = 0;  // chunks of the sequences before b
    int s_b = 0;   // chunks of sequence b
};

// Item v (< count_items) -> sequence b, head group hg, first key and key count.
template <bool HEAD_MAJOR>
__device__ __forceinline__ void decode_item(const DecodeParams &p, ItemCursor &c, int v, int &b, int &hg,
                                            int &start, int &n)
{
    const int lane = threadIdx.x & 31;
    const int u = v / p.n_hg;  // chunks of the sequences before b <= u < that + s_b
    if (u >= c.base + c.s_b) {
        int base = c.base + c.s_b, bb = c.b + 1;
        while (bb < p.B) {
            const int sb = (bb + lane < p.B) ? seq_chunks(p, bb + lane) : 0;
            int incl = sb;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += t;
            }
            const unsigned hit = __ballot_sync(0xffffffffu, base + incl > u);
            if (hit) {
                const int l = __ffs(hit) - 1;
                c.b = bb + l;
                c.s_b = __shfl_sync(0xffffffffu, sb, l);
                c.base = base + __shfl_sync(0xffffffffu, incl, l) - c.s_b;
                break;
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
            bb += 32;
        }
    }
    b = c.b;
    const int L = decode::clamp_len(p.seqlens[b], p.Nmax);
    if (HEAD_MAJOR) {
        const int r = v - c.base * p.n_hg;  // item of sequence b: r = hg * s_b + chunk
        hg = r / c.s_b;
        start = (r - hg * c.s_b) * decode::kChunk;
    } else {                                 // v = (base + chunk) * n_hg + hg
        hg = v - u * p.n_hg;
        start = (u - c.base) * decode::kChunk;
    }
    n = min(decode::kChunk, L - start);
}

// Split kernel for bf16 caches.  D: head dim (64 or 128).  RG: query heads per work item (<= 8,
// all of one KV head), the N = 8 columns of mma.sync m16n8k16 (columns RG .. 7 are zero):
// S^T = K Q^T per 16-key tile, O^T = V^T P^T per 16-dim tile, both with fp32
// accumulation; K and V fragments come from the swizzled stages through ldmatrix
// (transposed for V).
template <int D, int RG, bool PAGED>
__global__ void __launch_bounds__(decode::kThreads, decode::kCtasPerSm)
    fa_decode_split_kernel(const __grid_constant__ DecodeParams p)
{
    using namespace decode;
    using C = SplitCfg<D, RG>;
    static_assert(RG <= 8, "at most 8 query heads per item");
    constexpr int KSTEPS = D / 16;          // k-steps of S = Q K^T
    constexpr int VT = D / 16 / kWarps;     // 16-dim tiles of O^T per consumer warp
    static_assert(VT >= 1, "head dims per consumer warp");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float(*s_sm)[kChunk] = reinterpret_cast<float(*)[kChunk]>(smem + C::kScoreOff);
    float *m_sm = reinterpret_cast<float *>(smem + C::kMOff);
    float *l_sm = m_sm + RG;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *empty = full + C::kStages;
    uint64_t *group = empty + C::kStages;  // consumer-warp barrier
    int *stop_flag = reinterpret_cast<int *>(smem + C::kStopOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], kWarps);
        }
        ptx::mbar_init(group, kWarps);
        *stop_flag = 0;
        ptx::fence_barrier_init();
    }
    __syncthreads();
    // let the merge kernel (launched as a programmatic dependent) get scheduled early; it
    // waits for this whole grid to finish before it reads any partial
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const StopFlag sf{stop_flag, p.wait_limit_ns};
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int b = 0; b < p.B; ++b)
            if (p.seqlens[b] != clamp_len(p.seqlens[b], p.Nmax)) raise_error(kErrSeqlenRange);
    }

    if (warp == kWarps) {
        // ------------------------------------------------------------- producer
        const bool leader = ptx::elect_one();
        if (leader) {
            ptx::tma_prefetch_desc(&p.tm_k);
            ptx::tma_prefetch_desc(&p.tm_v);
        }
        uint32_t ring = 0;
        bool ok = true;
        const int n_items = count_items(p);
        // the cache is read once per call: its lines go first when L2 needs room (measured on
        // B200 after the prefill in one stream: 107 instead of 115 us on the decode workload,
        // whose reads no longer evict the prefill's output before it is written back)
        const uint64_t pol = ptx::l2_evict_first_policy();
        ItemCursor cur;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            int b, hg, start, n;
            decode_item<!PAGED>(p, cur, it, b, hg, start, n);
            const int g = hg * RG / p.R;
            const int plane = b * p.Hkv + g;
            // paged: lane i holds the physical page of the item's i-th logical page (an
            // item of kChunk keys spans at most kChunk / 16 + 1 <= 32 pages); an entry
            // outside the pool is reported and replaced by one past the pool's end, whose
            // copies read zeros
            int first_lp = 0, my_page = 0;
            if (PAGED) {
                first_lp = start / p.page_size;
                const int lp = first_lp + lane;
                if (lp <= (start + n - 1) / p.page_size &&
                    in_bounds((long long)b * p.max_pages + lp, (long long)p.B * p.max_pages)) {
                    my_page = p.block_table[(size_t)b * p.max_pages + lp];
                    if (my_page < 0 || my_page >= p.num_pages) {
                        raise_error(kErrPageRange);
                        my_page = p.num_pages;
                    }
                }
            }
            for (int pass = 0; pass < 2 && ok; ++pass) {
                const CUtensorMap *map = pass ? &p.tm_v : &p.tm_k;
                for (int t = 0; t * kSub < n; ++t) {
                    const uint32_t st = ring % C::kStages;
                    const uint32_t ph = (ring / C::kStages) & 1u;
                    if (!wait_warp(&empty[st], ph ^ 1u, sf)) { ok = false; break; }
                    if (p.selftest_no_full && ring == 0) {
                        // self-test: this stage is never filled (see DecodeParams)
                    } else if (PAGED) {
                        // only the boxes that hold keys of the sequence are copied (rows past
                        // it are masked or cleared by the consumers)
                        const int nbox = (min(kSub, n - t * kSub) + p.box_rows - 1) / p.box_rows;
                        if (leader) ptx::mbar_arrive_expect_tx(&full[st], nbox * p.box_rows * 128 * (D / 64));
                        for (int i = 0; i < nbox; ++i) {
                            const int key = start + t * kSub + i * p.box_rows;
                            const int lp = key / p.page_size;
                            const int page = __shfl_sync(0xffffffffu, my_page, lp - first_lp);
                            if (leader) {
#pragma unroll
                                for (int c = 0; c < (D / 64); ++c)
                                    ptx::tma_load_3d_hint(smem + st * C::kStageBytes + c * kBoxBytes + i * p.box_rows * 128,
                                                          map, &full[st], 64 * c, key - lp * p.page_size,
                                                          page * p.Hkv + g, pol);
                            }
                        }
                    } else if (leader) {
                        ptx::mbar_arrive_expect_tx(&full[st], C::kStageBytes);
#pragma unroll
                        for (int c = 0; c < (D / 64); ++c)
                            ptx::tma_load_3d_hint(smem + st * C::kStageBytes + c * kBoxBytes, map, &full[st],
                                                  64 * c, start + t * kSub, plane, pol);
                    }
                    __syncwarp();
                    ++ring;
                }
            }
        }
        // let every copy issued above land before the CTA can exit
        if (leader) {
            for (uint32_t st = 0; st < (uint32_t)C::kStages && st < ring; ++st) {
                const uint32_t last = ring - 1 - ((ring - 1 - st) % C::kStages);
                if (p.selftest_no_full && last == 0) continue;  // never issued
                const uint32_t par = (last / C::kStages) & 1u;
                const uint64_t t0 = ptx::globaltimer_ns();
                while (!ptx::mbar_test(&full[st], par))
                    if (ptx::globaltimer_ns() - t0 > p.wait_limit_ns) { raise_error(kErrTimeout); break; }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------- consumers
        const int gid = lane >> 2;   // fragment row (query head) / ldmatrix row group
        const int tig = lane & 3;    // thread in group
        const bool row_real = gid < RG;
        GroupBarrier gb{group, 0u};
        uint32_t ring = 0;
        // ldmatrix addressing: lane supplies row (lane & 7) of matrix (lane >> 3)
        const int lm_row = lane & 7;
        const int lm_mat = lane >> 3;
        const int n_items = count_items(p);
        ItemCursor cur;
        // The q rows of an item (the B operand of the K pass) are loaded one item ahead, so
        // that their latency overlaps the previous item's passes: r[2ks], r[2ks+1] = dims
        // 16ks + 2tig + {0,1}, 16ks + 8 + 2tig + {0,1}.
        auto load_q = [&](int qb_, int qhg, uint32_t (&r)[2 * KSTEPS]) {
            const long long qr = (long long)qb_ * p.Hq + qhg * RG + (row_real ? gid : 0);
            const bool use = row_real && in_bounds(qr, (long long)p.B * p.Hq);
            const uint32_t *qw = reinterpret_cast<const uint32_t *>(p.q + qr * D);
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                r[2 * ks] = use ? qw[8 * ks + tig] : 0u;
                r[2 * ks + 1] = use ? qw[8 * ks + 4 + tig] : 0u;
            }
        };
        int b = 0, hg = 0, start = 0, n = 0;
        uint32_t qraw[2 * KSTEPS];
        if ((int)blockIdx.x < n_items) {
            decode_item<!PAGED>(p, cur, blockIdx.x, b, hg, start, n);
            load_q(b, hg, qraw);
        }
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const int h0 = hg * RG;
            const int nit = it + gridDim.x;
            int nb = 0, nhg = 0, nstart = 0, nn = 0;
            uint32_t qnext[2 * KSTEPS];
            if (nit < n_items) {
                decode_item<!PAGED>(p, cur, nit, nb, nhg, nstart, nn);
                load_q(nb, nhg, qnext);
            }
            // The MMAs put the query heads in the N = 8 dimension (RG <= 8) and keys (K pass)
            // or head dims (V pass) in M = 16, so no MMA row is padding.
            // B operand of S^T = K Q^T: column gid = query head h0 + gid (zero beyond RG).
            // K step ks holds dims 16ks + 2tig + {0,1} and 16ks + 8 + 2tig + {0,1}.
            uint32_t qb[KSTEPS][2];
            const float sl = p.scale_log2;  // from the MMA result to log2-domain scores
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                qb[ks][0] = qraw[2 * ks];
                qb[ks][1] = qraw[2 * ks + 1];
            }
            const int hc0 = 2 * tig, hc1 = 2 * tig + 1;  // the heads of this lane's C columns
            bool ok = true;
            // ------------------------------------------------------------ K pass
            // warp w: S^T for keys 16w .. 16w+15 of each stage (A = 16 key rows of K)
            for (int t = 0; t * kSub < n; ++t) {
                const uint32_t st = ring % C::kStages;
                if (!wait_warp(&full[st], (ring / C::kStages) & 1u, sf)) { ok = false; break; }
                const uint32_t sbase = ptx::smem_addr(smem + st * C::kStageBytes);
                const int key0 = warp * 16;
                // two accumulators (even and odd K steps) halve the dependent MMA chain
                float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                // matrices: (keys 0-7 | 8-15) x (dims 16ks .. +7 | 16ks+8 .. +15)
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    uint32_t a[4];
                    ptx::ldsm_x4(sbase + stage_offset(key0 + (lm_mat & 1) * 8 + lm_row, 2 * ks + (lm_mat >> 1)),
                                 a[0], a[1], a[2], a[3]);
                    ptx::mma_16816_bf16(c[ks & 1], a, qb[ks][0], qb[ks][1]);
                }
                // c[.][0..1]: key key0 + gid, heads 2tig / 2tig+1; c[.][2..3]: key key0 + gid + 8
                const int ka = t * kSub + key0 + gid, kb8 = ka + 8;
                if (hc0 < RG) {
                    s_sm[hc0][ka] = ka < n ? (c[0][0] + c[1][0]) * sl : -INFINITY;
                    s_sm[hc0][kb8] = kb8 < n ? (c[0][2] + c[1][2]) * sl : -INFINITY;
                }
                if (hc1 < RG) {
                    s_sm[hc1][ka] = ka < n ? (c[0][1] + c[1][1]) * sl : -INFINITY;
                    s_sm[hc1][kb8] = kb8 < n ? (c[0][3] + c[1][3]) * sl : -INFINITY;
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&empty[st]);
                ++ring;
            }
            if (!ok || !gb.sync(sf)) break;
            // ------------------------------------------------------ chunk softmax
            for (int r = warp; r < RG; r += kWarps) {
                float mx = -INFINITY;
                for (int k = lane; k < n; k += 32) mx = fmaxf(mx, s_sm[r][k]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                float sum = 0.f;
                for (int k = lane; k < kChunk; k += 32) {
                    const float e = k < n ? ptx::ex2(s_sm[r][k] - mx) : 0.f;
                    s_sm[r][k] = e;
                    sum += e;
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                if (lane == 0) {
                    m_sm[r] = mx;
                    l_sm[r] = sum;
                }
            }
            if (!gb.sync(sf)) break;
            // ------------------------------------------------------------ V pass
            // warp w: O^T for head dims 16 VT w .. 16 VT (w+1) - 1, VT tiles of 16 (A = V^T).
            // Tile i rows = dims 16 (VT w + i) + (0..15).
            float acc[VT][4];
#pragma unroll
            for (int i = 0; i < VT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
            for (int t = 0; t * kSub < n; ++t) {
                const uint32_t st = ring % C::kStages;
                if (!wait_warp(&full[st], (ring / C::kStages) & 1u, sf)) { ok = false; break; }
                uint8_t *stage = smem + st * C::kStageBytes;
                const int rows = min(kSub, n - t * kSub);
                if (rows < kSub) {
                    // rows past the sequence hold whatever the cache holds there (or, paged,
                    // an earlier stage's data): clear them so that their zero weights cannot
                    // meet a non-finite value (and order these writes before the copy engine
                    // refills the stage)
                    for (int idx = threadIdx.x; idx < (kSub - rows) * C::kRowChunks; idx += 32 * kWarps) {
                        const int r = rows + idx / C::kRowChunks;
                        *reinterpret_cast<uint4 *>(stage + stage_offset(r, idx % C::kRowChunks)) = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                    if (!gb.sync(sf)) { ok = false; break; }
                }
                const uint32_t sbase = ptx::smem_addr(stage);
#pragma unroll
                for (int kb = 0; kb < kSub; kb += 16) {
                    // B operand: P^T, column gid = head gid, keys kb .. kb+15 (zero beyond RG)
                    uint32_t pb0 = 0u, pb1 = 0u;
                    if (row_real) {
                        const float2 p0 = *reinterpret_cast<const float2 *>(&s_sm[gid][t * kSub + kb + 2 * tig]);
                        const float2 p1 = *reinterpret_cast<const float2 *>(&s_sm[gid][t * kSub + kb + 8 + 2 * tig]);
                        pb0 = pack2_bf16(p0.x, p0.y);
                        pb1 = pack2_bf16(p1.x, p1.y);
                    }
#pragma unroll
                    for (int i = 0; i < VT; ++i) {
                        // matrices: (dims of the tile 0-7 | 8-15) x (keys kb..+7 | kb+8..+15)
                        const int chunk = 2 * (VT * warp + i) + (lm_mat & 1);
                        const int row = kb + (lm_mat >> 1) * 8 + lm_row;
                        uint32_t a[4];
                        ptx::ldsm_x4_trans(sbase + stage_offset(row, chunk), a[0], a[1], a[2], a[3]);
                        ptx::mma_16816_bf16(acc[i], a, pb0, pb1);
                    }
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&empty[st]);
                ++ring;
            }
            if (!ok) break;
            const int chunk = start / kChunk;
            // acc[i][0..1]: heads 2tig / 2tig+1 of tile row gid; acc[i][2..3]: of row gid + 8
            {
                const float f0 = hc0 < RG ? 1.f / l_sm[hc0] : 0.f;
                const float f1 = hc1 < RG ? 1.f / l_sm[hc1] : 0.f;
                const long long n_parts = (long long)p.B * p.Hq * p.S_max;  // partial rows in the workspace
                const long long r0p = ((long long)b * p.Hq + h0 + hc0) * p.S_max + chunk;
                const long long r1p = ((long long)b * p.Hq + h0 + hc1) * p.S_max + chunk;
                const bool w0 = hc0 < RG && in_bounds(r0p, n_parts), w1 = hc1 < RG && in_bounds(r1p, n_parts);
                float *dst0 = p.part_o + r0p * D;
                float *dst1 = p.part_o + r1p * D;
#pragma unroll
                for (int i = 0; i < VT; ++i) {
                    const int dim = 16 * (VT * warp + i) + gid;      // rows gid / gid + 8 = dims +0 / +8
                    if (w0) {
                        dst0[dim] = acc[i][0] * f0;
                        dst0[dim + 8] = acc[i][2] * f0;
                    }
                    if (w1) {
                        dst1[dim] = acc[i][1] * f1;
                        dst1[dim + 8] = acc[i][3] * f1;
                    }
                }
            }
            if (threadIdx.x < RG) {
                const long long rp = ((long long)b * p.Hq + h0 + threadIdx.x) * p.S_max + chunk;
                if (in_bounds(rp, (long long)p.B * p.Hq * p.S_max))
                    p.part_lse[rp] = m_sm[threadIdx.x] + ptx::lg2(l_sm[threadIdx.x]);
            }
            // scores and m/l are rewritten by the next item
            if (!gb.sync(sf)) break;
            b = nb;
            hg = nhg;
            start = nstart;
            n = nn;
#pragma unroll
            for (int i = 0; i < 2 * KSTEPS; ++i) qraw[i] = qnext[i];
        }
    }
    __syncthreads();
}

// Split kernel for FP8 (E4M3) caches, head dim 128: every consumer warp an independent worker.
// RG: query heads per work item (<= 8, all of one K/V head).  PAGED: the cache is a page pool
// addressed through the block table.
template <int RG, bool PAGED>
__global__ void __launch_bounds__(decode::kThreads, decode::kCtasPerSm)
    fa_decode_fp8_kernel(const __grid_constant__ DecodeParams p)
{
    using namespace decode;
    constexpr int D = 128;
    using C = WorkerCfg<RG>;
    constexpr int SK = kSK;
    constexpr int BOX = kStageBytes;
    constexpr int MT = SK / 16;         // 16-key M tiles of S^T per block
    constexpr int KSTEPS = D / 16;      // k-steps of S^T = K Q^T
    constexpr int VT = D / 16;          // 16-dim M tiles of O^T
    constexpr int PS = C::kPStride;
    static_assert(RG <= 8, "at most 8 query heads per item");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);  // [warp * 2 + (0: K, 1: V)]
    uint64_t *empty = full + 2 * kWarps;
    int *stop_flag = reinterpret_cast<int *>(smem + C::kStopOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * kWarps; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], 1);
        }
        *stop_flag = 0;
        ptx::fence_barrier_init();
    }
    __syncthreads();
    // let the merge kernel (launched as a programmatic dependent) get scheduled early; it
    // waits for this whole grid to finish before it reads any partial
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const StopFlag sf{stop_flag, p.wait_limit_ns};
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int b = 0; b < p.B; ++b)
            if (p.seqlens[b] != clamp_len(p.seqlens[b], p.Nmax)) raise_error(kErrSeqlenRange);
    }
    const int n_items = count_items(p);
    const int n_workers = (int)gridDim.x * kWarps;

    if (warp == kWarps) {
        // ------------------------------------------------------------- producer
        // Worker w's blocks, in order: K_0, V_0, K_1, V_1, ... of each of its items; K goes
        // to slot 0 of its ring and V to slot 1.  The whole warp runs the loop (every value
        // is warp-uniform; the per-worker state stays in registers because the loops over
        // workers are unrolled); one elected lane issues the copies.
        const bool leader = ptx::elect_one();
        if (leader) {
            ptx::tma_prefetch_desc(&p.tm_k);
            ptx::tma_prefetch_desc(&p.tm_v);
        }
        ItemCursor cur[kWarps];
        int it[kWarps] = {}, start[kWarps] = {}, n[kWarps] = {}, plane[kWarps] = {}, s[kWarps] = {}, g[kWarps] = {};
        int first_lp[kWarps] = {}, my_page[kWarps] = {};
        uint32_t kfill[kWarps] = {}, vfill[kWarps] = {};  // blocks copied to slot 0 (K) / 1 (V)
        // item it[w] of worker w: its keys, its plane, and (paged) the pages of its keys,
        // lane i holding the i-th (an item of kChunk keys spans at most kChunk / 16 + 1 <= 32
        // pages); an entry outside the pool is reported and replaced by one past the pool's
        // end, whose copies read zeros
        auto setup = [&](int w) {
            int b, hg;
            decode_item<false>(p, cur[w], it[w], b, hg, start[w], n[w]);
            g[w] = hg * RG / p.R;
            plane[w] = b * p.Hkv + g[w];
            s[w] = 0;
            if (PAGED) {
                first_lp[w] = start[w] / p.page_size;
                const int lp = first_lp[w] + lane;
                int pg = 0;
                if (lp <= (start[w] + n[w] - 1) / p.page_size &&
                    in_bounds((long long)b * p.max_pages + lp, (long long)p.B * p.max_pages)) {
                    pg = p.block_table[(size_t)b * p.max_pages + lp];
                    if (pg < 0 || pg >= p.num_pages) {
                        raise_error(kErrPageRange);
                        pg = p.num_pages;
                    }
                }
                my_page[w] = pg;
            }
        };
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            it[w] = w * (int)gridDim.x + (int)blockIdx.x;
            if (it[w] < n_items) setup(w);
        }
        bool ok = true;
        uint64_t idle_t0 = 0;
        uint32_t idle_n = 0;
        const uint64_t pol = ptx::l2_evict_first_policy();  // the cache is read once per call
        while (ok) {
            bool left = false, progressed = false;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                if (it[w] >= n_items) continue;
                left = true;
                const int v = s[w] & 1;
                const uint32_t f = v ? vfill[w] : kfill[w];
                if (!__all_sync(0xffffffffu, ptx::mbar_probe(&empty[2 * w + v], ((f & 1u) ^ 1u)))) continue;
                uint8_t *dst = smem + (2 * w + v) * kStageBytes;
                uint64_t *fb = &full[2 * w + v];
                const CUtensorMap *map = v ? &p.tm_v : &p.tm_k;
                const int key0 = start[w] + (s[w] >> 1) * SK;
                if (p.selftest_no_full && w == 0 && v == 0 && f == 0u) {
                    // self-test: worker 0's first K block is never filled (see DecodeParams)
                } else if (PAGED) {
                    // only the boxes that hold keys of the sequence are copied (rows past it
                    // are masked or cleared by the worker)
                    const int nbox = (min(SK, start[w] + n[w] - key0) + p.box_rows - 1) / p.box_rows;
                    if (leader) ptx::mbar_arrive_expect_tx(fb, nbox * p.box_rows * 128);
                    for (int i = 0; i < nbox; ++i) {
                        const int key = key0 + i * p.box_rows;
                        const int lp = key / p.page_size;
                        const int page = __shfl_sync(0xffffffffu, my_page[w], lp - first_lp[w]);
                        if (leader)
                            ptx::tma_load_3d_hint(dst + i * p.box_rows * 128, map, fb, 0, key - lp * p.page_size,
                                                  page * p.Hkv + g[w], pol);
                    }
                } else if (leader) {
                    // one box: 64 rows of 128 E4M3 bytes
                    ptx::mbar_arrive_expect_tx(fb, kStageBytes);
                    ptx::tma_load_3d_hint(dst, map, fb, 0, key0, plane[w], pol);
                }
                __syncwarp();
                if (v) vfill[w] = f + 1u;
                else kfill[w] = f + 1u;
                if (++s[w] == 2 * ((n[w] + SK - 1) / SK)) {
                    it[w] += n_workers;
                    if (it[w] < n_items) setup(w);
                }
                progressed = true;
            }
            if (!left) break;
            if (progressed) {
                idle_n = 0;
                continue;
            }
            // no ring had a free slot: bounded wait
            if (idle_n++ == 0) {
                idle_t0 = ptx::globaltimer_ns();
            } else if ((idle_n & 31u) == 0u) {
                int give_up = 0;
                if (lane == 0) {
                    if (sf.stopped()) {
                        give_up = 1;
                    } else if (ptx::globaltimer_ns() - idle_t0 > sf.limit_ns) {
                        raise_error(kErrTimeout);
                        sf.stop();
                        give_up = 1;
                    }
                }
                if (__shfl_sync(0xffffffffu, give_up, 0)) ok = false;
            }
        }
        // let every copy issued above land before the CTA can exit
        if (leader) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w)
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    const uint32_t f = v ? vfill[w] : kfill[w];
                    const bool withheld = p.selftest_no_full && w == 0 && v == 0 && f == 1u;
                    if (f > 0u && !withheld) {
                        const uint64_t t0 = ptx::globaltimer_ns();
                        while (!ptx::mbar_test(&full[2 * w + v], (f - 1u) & 1u))
                            if (ptx::globaltimer_ns() - t0 > p.wait_limit_ns) { raise_error(kErrTimeout); break; }
                    }
                }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------- worker
        const int gid = lane >> 2;   // C row group / B column (query head)
        const int tig = lane & 3;    // thread in group
        const bool row_real = gid < RG;
        const int hc0 = 2 * tig, hc1 = 2 * tig + 1;  // the heads of this lane's C columns
        // ldmatrix addressing: lane supplies row (lane & 7) of matrix (lane >> 3)
        const int lm_row = lane & 7;
        const int lm_mat = lane >> 3;
        const uint32_t k_saddr = ptx::smem_addr(smem + (2 * warp) * kStageBytes);
        const uint32_t v_saddr = k_saddr + kStageBytes;
        uint8_t *v_stage = smem + (2 * warp + 1) * kStageBytes;
        uint16_t *psm = reinterpret_cast<uint16_t *>(smem + C::kPOff + warp * C::kPBytes);  // [head][key]
        uint32_t kc = 0, vc = 0;  // K and V blocks consumed
        ItemCursor cur;
        // The q rows of an item (the B operand of S^T) and its k_scale are loaded one item
        // ahead, so that their latency overlaps the previous item: r[2ks], r[2ks+1] = dims
        // 16ks + 4tig + {0,1}, 16ks + 4tig + {2,3}.
        auto load_q = [&](int qb_, int qhg, uint32_t (&r)[2 * KSTEPS], float &ksc) {
            const long long qr = (long long)qb_ * p.Hq + qhg * RG + (row_real ? gid : 0);
            const bool use = row_real && in_bounds(qr, (long long)p.B * p.Hq);
            const __nv_bfloat16 *qrow = p.q + qr * D;
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                const uint2 raw = use ? *reinterpret_cast<const uint2 *>(qrow + 16 * ks + 4 * tig)
                                      : make_uint2(0u, 0u);
                r[2 * ks] = raw.x;
                r[2 * ks + 1] = raw.y;
            }
            ksc = in_bounds(qhg * RG / p.R, p.Hkv) ? p.k_scale[qhg * RG / p.R] : 0.f;
        };
        const int wid = warp * (int)gridDim.x + (int)blockIdx.x;
        int b = 0, hg = 0, start = 0, n = 0;
        uint32_t qraw[2 * KSTEPS];
        float kscale = 0.f;
        if (wid < n_items) {
            decode_item<false>(p, cur, wid, b, hg, start, n);
            load_q(b, hg, qraw, kscale);
        }
        for (int it = wid; it < n_items; it += n_workers) {
            const int h0 = hg * RG;
            const int g = h0 / p.R;
            const int nit = it + n_workers;
            int nb = 0, nhg = 0, nstart = 0, nn = 0;
            uint32_t qnext[2 * KSTEPS];
            float knext = 0.f;
            if (nit < n_items) {
                decode_item<false>(p, cur, nit, nb, nhg, nstart, nn);
                load_q(nb, nhg, qnext, knext);
            }
            // B operand of S^T = K Q^T (column gid = query head h0 + gid, zero beyond RG) and
            // the factors from the MMA result to log2-domain scores of heads 2tig, 2tig+1
            uint32_t qb[KSTEPS][2];
            float sl0 = p.scale_log2, sl1 = p.scale_log2;
            float qv[KSTEPS][4];
            float amax = 0.f;
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                qv[ks][0] = __uint_as_float(qraw[2 * ks] << 16);
                qv[ks][1] = __uint_as_float(qraw[2 * ks] & 0xffff0000u);
                qv[ks][2] = __uint_as_float(qraw[2 * ks + 1] << 16);
                qv[ks][3] = __uint_as_float(qraw[2 * ks + 1] & 0xffff0000u);
#pragma unroll
                for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(qv[ks][e]));
            }
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            // 2^e with amax * 2^e in [2^14, 2^15); e kept within the normal range
            int e = 0;
            if (amax > 0.f) e = 14 - (((int)(__float_as_uint(amax) >> 23) & 0xff) - 127);
            e = max(-120, min(120, e));
            const float up = __uint_as_float((uint32_t)(127 + e) << 23);
            const float down = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                qb[ks][0] = ptx::pack_f16x2(qv[ks][0] * up, qv[ks][1] * up);
                qb[ks][1] = ptx::pack_f16x2(qv[ks][2] * up, qv[ks][3] * up);
            }
            const float sl_own = p.scale_log2 * kscale * down;  // head gid
            sl0 = __shfl_sync(0xffffffffu, sl_own, 8 * tig);            // head 2tig
            sl1 = __shfl_sync(0xffffffffu, sl_own, 8 * tig + 4);        // head 2tig+1
            // online softmax state of heads 2tig, 2tig+1 (l: this lane's part of the sum) and
            // O^T (acc[i]: head dims of tile i x heads 2tig, 2tig+1)
            float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
            float acc[VT][4];
#pragma unroll
            for (int i = 0; i < VT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
            bool ok = true;
            const int nblk = (n + SK - 1) / SK;
            for (int t = 0; t < nblk; ++t) {
                // ---------------------------------------------- S^T for keys t*SK ..
                if (!wait_warp(&full[2 * warp], kc & 1u, sf)) { ok = false; break; }
                float c[MT][4];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    c[mt][0] = c[mt][1] = c[mt][2] = c[mt][3] = 0.f;
                    // matrices: (keys 0-7 | 8-15 of the tile) x (16-byte chunk 2j | 2j+1); a
                    // lane's register = dims 4tig .. 4tig+3 of key gid (or gid + 8)
#pragma unroll
                    for (int j = 0; j < KSTEPS / 2; ++j) {
                        uint32_t r[4];
                        ptx::ldsm_x4(k_saddr + stage_offset<BOX>(16 * mt + (lm_mat & 1) * 8 + lm_row, 2 * j + (lm_mat >> 1)),
                                     r[0], r[1], r[2], r[3]);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t lo = r[2 * h], hi = r[2 * h + 1];
                            uint32_t a[4];
                            e4m3_halves_f16x2(lo, a[0], a[2]);  // dims (0, 1) and (2, 3) of key gid
                            e4m3_halves_f16x2(hi, a[1], a[3]);  // ... of key gid + 8
                            ptx::mma_16816_f16(c[mt], a, qb[2 * j + h][0], qb[2 * j + h][1]);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&empty[2 * warp]);
                ++kc;
                // ------------------------------------------------- online softmax
                // c[mt][0..1]: key 16mt + gid, heads 2tig / 2tig+1; c[mt][2..3]: key + 8
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const int ka = t * SK + 16 * mt + gid;
                    c[mt][0] = ka < n ? c[mt][0] * sl0 : -INFINITY;
                    c[mt][1] = ka < n ? c[mt][1] * sl1 : -INFINITY;
                    c[mt][2] = ka + 8 < n ? c[mt][2] * sl0 : -INFINITY;
                    c[mt][3] = ka + 8 < n ? c[mt][3] * sl1 : -INFINITY;
                    mx0 = ptx::max3(mx0, c[mt][0], c[mt][2]);
                    mx1 = ptx::max3(mx1, c[mt][1], c[mt][3]);
                }
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                // every block holds at least one key of the item, so mx is finite; on the
                // first block m is -inf and the factor is 0
                const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                const float al0 = ptx::ex2(m0 - mn0), al1 = ptx::ex2(m1 - mn1);
                m0 = mn0;
                m1 = mn1;
                l0 *= al0;
                l1 *= al1;
#pragma unroll
                for (int i = 0; i < VT; ++i) {
                    acc[i][0] *= al0;
                    acc[i][2] *= al0;
                    acc[i][1] *= al1;
                    acc[i][3] *= al1;
                }
                // P (fp16, the type of the V operand) into this warp's tile, [head][key]
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const float p0 = ptx::ex2(c[mt][0] - m0), p1 = ptx::ex2(c[mt][1] - m1);
                    const float p2 = ptx::ex2(c[mt][2] - m0), p3 = ptx::ex2(c[mt][3] - m1);
                    l0 += p0 + p2;
                    l1 += p1 + p3;
                    const uint32_t w01 = ptx::pack_f16x2(p0, p1);
                    const uint32_t w23 = ptx::pack_f16x2(p2, p3);
                    const int kl = 16 * mt + gid;
                    psm[hc0 * PS + kl] = (uint16_t)(w01 & 0xffffu);
                    psm[hc1 * PS + kl] = (uint16_t)(w01 >> 16);
                    psm[hc0 * PS + kl + 8] = (uint16_t)(w23 & 0xffffu);
                    psm[hc1 * PS + kl + 8] = (uint16_t)(w23 >> 16);
                }
                __syncwarp();
                // ------------------------------------------------- O^T += V^T P^T
                if (!wait_warp(&full[2 * warp + 1], vc & 1u, sf)) { ok = false; break; }
                const int rows = min(SK, n - t * SK);
                if (rows < SK) {
                    // rows past the sequence hold whatever the cache (or, paged, an earlier
                    // block) holds there: clear them so that their zero weights cannot meet a
                    // non-finite value, and order these writes before the copy engine
                    // refills the slot
                    for (int idx = lane; idx < (SK - rows) * 8; idx += 32) {
                        const int r = rows + idx / 8;
                        *reinterpret_cast<uint4 *>(v_stage + stage_offset<BOX>(r, idx % 8)) =
                            make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                }
                // Not unrolled: the worker loop body stays small enough for the instruction
                // cache (measured on B200: +3% on the FP8 decode workload against the
                // unrolled loop; not unrolling the K pass as well loses 4%)
#pragma unroll 1
                for (int kb = 0; kb < SK; kb += 16) {
                    // B operand: P^T, column gid = head gid, keys kb .. kb+15
                    const uint32_t pb0 = *reinterpret_cast<const uint32_t *>(&psm[gid * PS + kb + 2 * tig]);
                    const uint32_t pb1 = *reinterpret_cast<const uint32_t *>(&psm[gid * PS + kb + 8 + 2 * tig]);
                    // matrices: (keys kb..+7 | kb+8..+15) x (16-byte chunk 2j | 2j+1); a lane
                    // gets bytes {V[2tig][2gid], V[2tig][2gid+1], V[2tig+1][2gid],
                    // V[2tig+1][2gid+1]} of its matrix: bytes (0, 2) are the key pair of
                    // dim 2gid, bytes (1, 3) that of dim 2gid+1
#pragma unroll
                    for (int j = 0; j < VT / 2; ++j) {
                        uint32_t r[4];
                        ptx::ldsm_x4_trans(v_saddr + stage_offset<BOX>(kb + (lm_mat & 1) * 8 + lm_row, 2 * j + (lm_mat >> 1)),
                                           r[0], r[1], r[2], r[3]);
#pragma unroll
                        for (int i2 = 0; i2 < 2; ++i2) {
                            const uint32_t klo = r[2 * i2], khi = r[2 * i2 + 1];
                            // bytes (0, 2, 1, 3): the even dim's key pair, then the odd dim's
                            uint32_t a[4];
                            e4m3_halves_f16x2(__byte_perm(klo, 0u, 0x3120u), a[0], a[1]);
                            e4m3_halves_f16x2(__byte_perm(khi, 0u, 0x3120u), a[2], a[3]);
                            ptx::mma_16816_f16(acc[2 * j + i2], a, pb0, pb1);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&empty[2 * warp + 1]);
                ++vc;
            }
            if (!ok) break;
            // --------------------------------------------------------- item result
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, off);
                l1 += __shfl_xor_sync(0xffffffffu, l1, off);
            }
            const int chunk = start / kChunk;
            // acc[i][0..1]: heads 2tig / 2tig+1 of tile row gid; acc[i][2..3]: of row gid + 8
            const float vsc = in_bounds(g, p.Hkv) ? p.v_scale[g] : 0.f;
            const float f0 = vsc / l0;
            const float f1 = vsc / l1;
            const long long n_parts = (long long)p.B * p.Hq * p.S_max;  // partial rows in the workspace
            const long long r0p = ((long long)b * p.Hq + h0 + hc0) * p.S_max + chunk;
            const long long r1p = ((long long)b * p.Hq + h0 + hc1) * p.S_max + chunk;
            const bool w0 = hc0 < RG && in_bounds(r0p, n_parts), w1 = hc1 < RG && in_bounds(r1p, n_parts);
            float *dst0 = p.part_o + r0p * D;
            float *dst1 = p.part_o + r1p * D;
#pragma unroll
            for (int i = 0; i < VT; ++i) {
                const int dim = 16 * i + 2 * gid;  // rows gid / gid + 8 = dims +0 / +1
                if (w0) *reinterpret_cast<float2 *>(dst0 + dim) = make_float2(acc[i][0] * f0, acc[i][2] * f0);
                if (w1) *reinterpret_cast<float2 *>(dst1 + dim) = make_float2(acc[i][1] * f1, acc[i][3] * f1);
            }
            if (gid == 0) {
                if (w0) p.part_lse[r0p] = m0 + ptx::lg2(l0);
                if (w1) p.part_lse[r1p] = m1 + ptx::lg2(l1);
            }
            b = nb;
            hg = nhg;
            start = nstart;
            n = nn;
            kscale = knext;
#pragma unroll
            for (int i = 0; i < 2 * KSTEPS; ++i) qraw[i] = qnext[i];
        }
    }
    __syncthreads();
}

// One CTA of kMergeWarps warps per (query head, sequence).  Every warp finds the largest
// partial log2-sum-exp M (lanes stride over the S partials); warp w then accumulates the
// weighted partial outputs of splits w, w + kMergeWarps, ... with each lane owning D/32
// consecutive elements (one vector load per split); the warps' sums are added in shared
// memory.
constexpr int kMergeWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kMergeWarps) fa_decode_merge_kernel(const __grid_constant__ DecodeParams p)
{
    using namespace decode;
    // wait until the split kernel's partials are complete and visible (no-op when this
    // kernel was not launched as a programmatic dependent)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int EPL = D / 32;  // output elements per lane
    __shared__ float red[kMergeWarps][D];
    __shared__ float den_sm[kMergeWarps];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const size_t bh = blockIdx.x;
    const int b = (int)(bh / p.Hq);
    if (!in_bounds((long long)bh, (long long)p.B * p.Hq)) return;  // (whole CTA: uniform)
    const int L = clamp_len(p.seqlens[b], p.Nmax);
    const int S = (L + kChunk - 1) / kChunk;
    if (!in_bounds(S, (long long)p.S_max + 1)) return;
    const float *pl = p.part_lse + bh * p.S_max;
    const float *po = p.part_o + bh * p.S_max * D;
    if (S == 0) {
        if (threadIdx.x < D) {
            if (p.o_f32) p.o_f32[bh * D + threadIdx.x] = 0.f;
            else p.o[bh * D + threadIdx.x] = __float2bfloat16_rn(0.f);
        }
        if (threadIdx.x == 0 && p.lse) p.lse[bh] = -INFINITY;
        return;
    }
    float M = -INFINITY;
    for (int s = lane; s < S; s += 32) M = fmaxf(M, pl[s]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float den = 0.f;
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
#pragma unroll 4
    for (int s = warp; s < S; s += kMergeWarps) {
        const float w = ptx::ex2(pl[s] - M);
        den += w;
        const float *src = po + (size_t)s * D + lane * EPL;
        if constexpr (EPL == 4) {
            const float4 x = *reinterpret_cast<const float4 *>(src);
            acc[0] = fmaf(w, x.x, acc[0]);
            acc[1] = fmaf(w, x.y, acc[1]);
            acc[2] = fmaf(w, x.z, acc[2]);
            acc[3] = fmaf(w, x.w, acc[3]);
        } else {
            const float2 x = *reinterpret_cast<const float2 *>(src);
            acc[0] = fmaf(w, x.x, acc[0]);
            acc[1] = fmaf(w, x.y, acc[1]);
        }
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) red[warp][lane * EPL + e] = acc[e];
    if (lane == 0) den_sm[warp] = den;
    __syncthreads();
    if (threadIdx.x < D) {
        float t = 0.f, dsum = 0.f;
#pragma unroll
        for (int w = 0; w < kMergeWarps; ++w) {
            t += red[w][threadIdx.x];
            dsum += den_sm[w];
        }
        if (p.o_f32) p.o_f32[bh * D + threadIdx.x] = t / dsum;
        else p.o[bh * D + threadIdx.x] = __float2bfloat16_rn(t / dsum);
        if (threadIdx.x == 0 && p.lse) p.lse[bh] = (M + ptx::lg2(dsum)) * kLn2;
    }
}

// Merge of P partial results computed elsewhere (for instance on other GPUs, each over
// its own part of the keys): the log-sum-exp merge above with natural-log inputs.
//   o_parts (P, rows, D) fp32, lse_parts (P, rows) natural log (-inf: no keys);
//   o (rows, D) bf16 or o_f32 fp32; lse (rows) natural log, may be null.
// One warp per row; lane owns D/32 consecutive elements.
struct MergeLseParams {
    const float *o_parts;
    const float *lse_parts;
    __nv_bfloat16 *o;
    float *o_f32;
    float *lse;
    int P, rows;
};

constexpr int kMergeLseWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kMergeLseWarps) fa_merge_lse_kernel(const __grid_constant__ MergeLseParams m)
{
    constexpr int EPL = D / 32;
    constexpr float kLog2e = 1.4426950408889634f;
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kMergeLseWarps + (threadIdx.x >> 5);
    if (row >= m.rows) return;
    float M = -INFINITY;
    for (int q = lane; q < m.P; q += 32) M = fmaxf(M, m.lse_parts[(size_t)q * m.rows + row]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    float den = 0.f;
    if (M != -INFINITY) {
        for (int q = 0; q < m.P; ++q) {
            const float l = m.lse_parts[(size_t)q * m.rows + row];
            if (l == -INFINITY) continue;  // a part with no keys: weight 0
            const float w = ptx::ex2((l - M) * kLog2e);
            den += w;
            const float *src = m.o_parts + ((size_t)q * m.rows + row) * D + lane * EPL;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, src[e], acc[e]);
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        const size_t i = (size_t)row * D + lane * EPL + e;
        if (m.o_f32) m.o_f32[i] = acc[e] * inv;
        else m.o[i] = __float2bfloat16_rn(acc[e] * inv);
    }
    if (lane == 0 && m.lse) m.lse[row] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace fa
