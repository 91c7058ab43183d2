// fa_decode_sm100.cuh -- split-KV decode over a KV cache, with a log-sum-exp merge.
//
// Decode (one new query row per sequence) reads the whole cache every step and does
// only 4 flops per byte, so it is bound by HBM bandwidth (youngju.dev "attention
// variants", section 7).  The cache of one (sequence, key/value head) is contiguous, so
// it is cut into chunks of kChunk keys that independent CTAs stream in parallel:
//
//   split kernel, one CTA per (chunk, group of RG query heads of one KV head, sequence):
//     K pass: each lane reads one 16-byte slice of a key row (fully coalesced, several
//             loads in flight), scores for the RG heads are reduced across the lanes of
//             the row; scores (pre-multiplied by scale*log2 e) go to shared memory.
//     softmax of the chunk: max, p = 2^(s - max), sum.
//     V pass: the same slicing over value rows, O_part += p * v in fp32.
//     writes the normalised partial output and its log2-sum-exp to the workspace.
//   merge kernel, one CTA per (head, sequence): M = max of the partial log-sum-exps,
//     w_s = 2^(lse_s - M), o = sum_s w_s o_s / sum_s w_s, lse = M + log2 sum_s w_s.
// The merge is the same rescaling the online softmax applies between key blocks
// (youngju.dev section 3), applied across chunks.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "fa_common.cuh"
#include "ptx_sm100.cuh"

namespace fa {

struct DecodeParams {
    const __nv_bfloat16 *q;   // (B, Hq, D)
    const __nv_bfloat16 *kc;  // (B, Hkv, Nmax, D)
    const __nv_bfloat16 *vc;  // (B, Hkv, Nmax, D)
    const int *seqlens;       // (B)
    float *part_o;            // (B, Hq, S_max, D)  normalised partial outputs
    float *part_lse;          // (B, Hq, S_max)     partial log2-sum-exp (scaled scores)
    __nv_bfloat16 *o;         // (B, Hq, D)
    float *lse;               // (B, Hq) natural log, may be null
    int B, Hq, Hkv, Nmax, R, S_max;
    float scale_log2;
};

namespace decode {

constexpr int kChunk = 256;
constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 8;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ int clamp_len(int L, int Nmax)
{
    return L < 0 ? 0 : (L > Nmax ? Nmax : L);
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8])
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void unpack8x2(const uint4 &u, float2 (&f)[4])
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

// Sums V values per lane over the LPK lanes that share one key row and scatters the
// results: after the call lane `sub` holds, in a[0], the full sum of value head_of(sub).
// Levels with more than one value left halve the values (a lane keeps one half and adds
// its partner's copy of that half), the remaining levels are plain butterflies.
template <int V, int LPK>
__device__ __forceinline__ void reduce_scatter(float (&a)[V], int sub)
{
    int n = V;
#pragma unroll
    for (int off = LPK / 2; off >= 1; off >>= 1) {
        if (n > 1) {
            const int half = n >> 1;
            const bool upper = (sub & off) != 0;
#pragma unroll
            for (int i = 0; i < V / 2; ++i) {
                if (i < half) {
                    const float send = upper ? a[i] : a[i + half];
                    const float keep = upper ? a[i + half] : a[i];
                    a[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            n = half;
        } else {
            a[0] += __shfl_xor_sync(0xffffffffu, a[0], off);
        }
    }
}

// Which value lane `sub` holds after reduce_scatter<V, LPK>, and whether it is the one
// lane (of the group holding that value) that writes it.
template <int V, int LPK>
__device__ __forceinline__ int scatter_head(int sub, bool &writer)
{
    int head = 0, n = V, low_mask = 0;
#pragma unroll
    for (int off = LPK / 2; off >= 1; off >>= 1) {
        if (n > 1) {
            n >>= 1;
            if (sub & off) head += n;
        } else {
            low_mask |= off;
        }
    }
    writer = (sub & low_mask) == 0;
    return head;
}

__device__ __forceinline__ uint4 ldg_stream(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

}  // namespace decode

// D: head dim (64 or 128).  RG: query heads per CTA (all of one KV head).
template <int D, int RG>
__global__ void __launch_bounds__(decode::kThreads)
    fa_decode_split_kernel(const __grid_constant__ DecodeParams p)
{
    using namespace decode;
    constexpr int LPK = D / 8;      // lanes per key row (16 bytes each)
    constexpr int KPW = 32 / LPK;   // key rows per warp instruction
    constexpr int KPI = KPW * kWarps;  // key rows per CTA instruction

    __shared__ float s_sm[RG][kChunk];
    __shared__ float red[kWarps][RG][D];
    __shared__ float m_sm[RG], l_sm[RG];

    // let the merge kernel (launched as a programmatic dependent) get scheduled early; it
    // waits for this whole grid to finish before it reads any partial
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int chunk = blockIdx.x;
    const int h0 = blockIdx.y * RG;
    const int b = blockIdx.z;
    const int raw = p.seqlens[b];
    const int L = clamp_len(raw, p.Nmax);
    if (raw != L && chunk == 0 && blockIdx.y == 0 && threadIdx.x == 0) raise_error(kErrSeqlenRange);
    const int start = chunk * kChunk;
    if (start >= L) return;
    const int n = min(kChunk, L - start);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPK;   // which 16-byte slice of the row
    const int kk = lane / LPK;    // which row of the warp's group
    const int g = h0 / p.R;

    const size_t plane = ((size_t)b * p.Hkv + g) * (size_t)p.Nmax + (size_t)start;
    const __nv_bfloat16 *kbase = p.kc + plane * D + sub * 8;
    const __nv_bfloat16 *vbase = p.vc + plane * D + sub * 8;

    float2 qf[RG][4];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p.q + ((size_t)b * p.Hq + h0 + r) * D + sub * 8);
        unpack8x2(u, qf[r]);
#pragma unroll
        for (int e = 0; e < 4; ++e) qf[r][e] = __fmul2_rn(qf[r][e], make_float2(p.scale_log2, p.scale_log2));
    }
    bool writer;
    const int my_head = scatter_head<RG, LPK>(sub, writer);

    // ---------------------------------------------------------------- K pass
    for (int base = 0; base < n; base += KPI * kUnroll) {
        uint4 kr[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int key = base + u * KPI + warp * KPW + kk;
            kr[u] = key < n ? ldg_stream(kbase + (size_t)key * D) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int key = base + u * KPI + warp * KPW + kk;
            float2 kf[4];
            unpack8x2(kr[u], kf);
            float acc[RG];
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                float2 a = __fmul2_rn(qf[r][0], kf[0]);
#pragma unroll
                for (int e = 1; e < 4; ++e) a = __ffma2_rn(qf[r][e], kf[e], a);
                acc[r] = a.x + a.y;
            }
            reduce_scatter<RG, LPK>(acc, sub);
            if (writer && key < n) s_sm[my_head][key] = acc[0];
        }
    }
    __syncthreads();

    // ------------------------------------------------------- chunk softmax
    for (int r = warp; r < RG; r += kWarps) {
        float mx = -INFINITY;
        for (int k = lane; k < n; k += 32) mx = fmaxf(mx, s_sm[r][k]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float sum = 0.f;
        for (int k = lane; k < n; k += 32) {
            const float e = ptx::ex2(s_sm[r][k] - mx);
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
    __syncthreads();

    // ---------------------------------------------------------------- V pass
    float2 acc[RG][4];
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][e] = make_float2(0.f, 0.f);
    for (int base = 0; base < n; base += KPI * kUnroll) {
        uint4 vr[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int key = base + u * KPI + warp * KPW + kk;
            vr[u] = key < n ? ldg_stream(vbase + (size_t)key * D) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int key = base + u * KPI + warp * KPW + kk;
            if (key < n) {
                float2 vf[4];
                unpack8x2(vr[u], vf);
#pragma unroll
                for (int r = 0; r < RG; ++r) {
                    const float pr = s_sm[r][key];
                    const float2 p2 = make_float2(pr, pr);
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[r][e] = __ffma2_rn(p2, vf[e], acc[r][e]);
                }
            }
        }
    }
    // rows handled by different lanes of a warp -> lanes with kk == 0
#pragma unroll
    for (int off = LPK; off < 32; off <<= 1)
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[r][e].x += __shfl_xor_sync(0xffffffffu, acc[r][e].x, off);
                acc[r][e].y += __shfl_xor_sync(0xffffffffu, acc[r][e].y, off);
            }
    if (kk == 0) {
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                red[warp][r][sub * 8 + 2 * e] = acc[r][e].x;
                red[warp][r][sub * 8 + 2 * e + 1] = acc[r][e].y;
            }
    }
    __syncthreads();

    for (int idx = threadIdx.x; idx < RG * D; idx += kThreads) {
        const int r = idx / D;
        const int e = idx - r * D;
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) t += red[w][r][e];
        p.part_o[(((size_t)b * p.Hq + h0 + r) * p.S_max + chunk) * D + e] = t / l_sm[r];
    }
    if (threadIdx.x < RG)
        p.part_lse[((size_t)b * p.Hq + h0 + threadIdx.x) * p.S_max + chunk] =
            m_sm[threadIdx.x] + ptx::lg2(l_sm[threadIdx.x]);
}

// One CTA of kMergeWarps warps per (query head, sequence).  Every warp finds the largest
// partial log2-sum-exp M (lanes stride over the S partials); warp w then accumulates the
// weighted partial outputs of splits w, w + kMergeWarps, ... with each lane owning D/32
// consecutive elements; the warps' sums are added in shared memory.
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
    const int L = clamp_len(p.seqlens[b], p.Nmax);
    const int S = (L + kChunk - 1) / kChunk;
    const float *pl = p.part_lse + bh * p.S_max;
    const float *po = p.part_o + bh * p.S_max * D;
    if (S == 0) {
        if (threadIdx.x < D) p.o[bh * D + threadIdx.x] = __float2bfloat16_rn(0.f);
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
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, src[e], acc[e]);
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
        p.o[bh * D + threadIdx.x] = __float2bfloat16_rn(t / dsum);
        if (threadIdx.x == 0 && p.lse) p.lse[bh] = (M + ptx::lg2(dsum)) * kLn2;
    }
}

}  // namespace fa
