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

    float qf[RG][8];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p.q + ((size_t)b * p.Hq + h0 + r) * D + sub * 8);
        unpack8(u, qf[r]);
#pragma unroll
        for (int e = 0; e < 8; ++e) qf[r][e] *= p.scale_log2;
    }

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
            float kf[8];
            unpack8(kr[u], kf);
            float acc[RG];
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) a = fmaf(qf[r][e], kf[e], a);
                acc[r] = a;
            }
#pragma unroll
            for (int off = 1; off < LPK; off <<= 1)
#pragma unroll
                for (int r = 0; r < RG; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], off);
            if (sub == 0 && key < n) {
#pragma unroll
                for (int r = 0; r < RG; ++r) s_sm[r][key] = acc[r];
            }
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
    float acc[RG][8];
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
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
                float vf[8];
                unpack8(vr[u], vf);
#pragma unroll
                for (int r = 0; r < RG; ++r) {
                    const float pr = s_sm[r][key];
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[r][e] = fmaf(pr, vf[e], acc[r][e]);
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
            for (int e = 0; e < 8; ++e) acc[r][e] += __shfl_xor_sync(0xffffffffu, acc[r][e], off);
    if (kk == 0) {
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int e = 0; e < 8; ++e) red[warp][r][sub * 8 + e] = acc[r][e];
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

// One CTA per (query head, sequence); thread e owns output element e.
template <int D>
__global__ void __launch_bounds__(128) fa_decode_merge_kernel(const __grid_constant__ DecodeParams p)
{
    using namespace decode;
    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int L = clamp_len(p.seqlens[b], p.Nmax);
    const int S = (L + kChunk - 1) / kChunk;
    const size_t bh = (size_t)b * p.Hq + h;
    const float *pl = p.part_lse + bh * p.S_max;
    const float *po = p.part_o + bh * p.S_max * D;
    if (S == 0) {
        if (threadIdx.x < D) p.o[bh * D + threadIdx.x] = __float2bfloat16_rn(0.f);
        if (threadIdx.x == 0 && p.lse) p.lse[bh] = -INFINITY;
        return;
    }
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, pl[s]);
    float den = 0.f, num = 0.f;
    const int e = threadIdx.x;
    for (int s = 0; s < S; ++s) {
        const float w = ptx::ex2(pl[s] - M);
        den += w;
        if (e < D) num = fmaf(w, po[(size_t)s * D + e], num);
    }
    if (e < D) p.o[bh * D + e] = __float2bfloat16_rn(num / den);
    if (e == 0 && p.lse) p.lse[bh] = (M + ptx::lg2(den)) * kLn2;
}

}  // namespace fa
