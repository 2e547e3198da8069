// Merge of split-KV parts (ruDNN "merge FP32 statistics"; alice-llm `lse_combine`).
// Part i of a row holds its normalised output o_i and logsumexp lse_i over its keys; the
// merged lse is logsumexp_i(lse_i) and the merged output is sum_i exp(lse_i - lse) * o_i.
// Parts without keys carry lse_i = -inf and weight 0; a row whose parts are all empty gets
// out = 0 and lse = -inf.
//
// One warp per (query, head, up to 512 output columns): the weights go to shared memory once per
// row; each lane owns four consecutive columns (float4) of each of the row's (up to four)
// 128-column chunks and walks the parts two or four at a time (eight loads in flight). The merge is
// a short, latency-bound read of parts the attention kernel has just written: the first parts'
// rows are requested before the weights are known, and the registers stay low enough for one wave.
#include "device_common.cuh"

namespace pa {

constexpr int kCombineWarps = 4;
constexpr int kCombineMaxSplits = 1024;
constexpr int kCombineCols = 512;  // output columns per warp at most (wider rows spread over more CTAs)

template <typename T>
__device__ __forceinline__ void store4(T* dst, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* dst, float4 v) {
    *reinterpret_cast<float4*>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
    uint2 u;
    u.x = pack2<__nv_bfloat16>(v.x, v.y);
    u.y = pack2<__nv_bfloat16>(v.z, v.w);
    *reinterpret_cast<uint2*>(dst) = u;
}
template <>
__device__ __forceinline__ void store4<__half>(__half* dst, float4 v) {
    uint2 u;
    u.x = pack2<__half>(v.x, v.y);
    u.y = pack2<__half>(v.z, v.w);
    *reinterpret_cast<uint2*>(dst) = u;
}

__device__ __forceinline__ void fma4(float4& a, float w, const float4 b) {
    a.x = fmaf(w, b.x, a.x);
    a.y = fmaf(w, b.y, a.y);
    a.z = fmaf(w, b.z, a.z);
    a.w = fmaf(w, b.w, a.w);
}

template <typename T, int NJ>
__global__ void __launch_bounds__(kCombineWarps * 32, 7) combine_kernel(const AttnParams p) {
    // parts in flight per lane: four with one 128-column chunk, two with two or four chunks (at
    // most eight float4 loads), so that the kernel fits 72 registers and seven CTAs per SM, and the
    // usual grids one wave
    constexpr int PF = NJ >= 2 ? 2 : 4;
    __shared__ float wts[kCombineWarps][kCombineMaxSplits];
    const CombineUnit cu = p.cunits[blockIdx.x];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y * kCombineWarps + warp;
    if (h >= p.hq) return;
    const int c_lo = blockIdx.z * kCombineCols;  // this warp's output columns [c_lo, c_hi)
    const int c_hi = min(p.dv, c_lo + kCombineCols);
    const int n = cu.nsplit;
    const float* ls = p.ws_lse + (int64_t)cu.part_base * p.hq + h;
    const float* op = p.ws_o + ((int64_t)cu.part_base * p.hq + h) * p.dv;
    const int64_t step = (int64_t)p.hq * p.dv;
    const float kLog2e = 1.4426950408889634f;
    const bool vec = (p.dv & 3) == 0;
    // chunk j: columns c_lo + 128 j + 4 lane .. + 3 (when inside [c_lo, c_hi))
    bool on[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) on[j] = vec && c_lo + 128 * j + lane * 4 < c_hi;
    const float* base = op + c_lo + lane * 4;
    float4 b[PF][NJ];
    auto load = [&](int i0) {
#pragma unroll
        for (int x = 0; x < PF; ++x)
#pragma unroll
            for (int j = 0; j < NJ; ++j)
                b[x][j] = on[j] && i0 + x < n ? *reinterpret_cast<const float4*>(base + (i0 + x) * step + 128 * j)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    // the first parts' rows are requested together with the logsumexps: they do not depend on
    // the weights. Up to 32 parts: each lane keeps its part's logsumexp, so the max and the sum
    // need one round of loads; more parts are read again for the sum.
    load(0);
    const float my_l = lane < n ? ls[(int64_t)lane * p.hq] : neg_inf();
    float m = my_l;
    for (int i = lane + 32; i < n; i += 32) m = fmaxf(m, ls[(int64_t)i * p.hq]);
    m = warp_max(m);
    const int64_t row = (int64_t)cu.query * p.hq + h;
    T* o = static_cast<T*>(p.out) + row * p.dv;
    if (m == neg_inf()) {
        for (int c = c_lo + lane; c < c_hi; c += 32) o[c] = from_f32<T>(0.f);
        if (lane == 0 && blockIdx.z == 0) p.lse[row] = m;
        return;
    }
    float sum = lane < n ? fast_exp2((my_l - m) * kLog2e) : 0.f;
    for (int i = lane + 32; i < n; i += 32) sum += fast_exp2((ls[(int64_t)i * p.hq] - m) * kLog2e);
    sum = warp_sum(sum);
    const float lse = m + __logf(sum);
    if (lane < n) wts[warp][lane] = fast_exp2((my_l - lse) * kLog2e);
    for (int i = lane + 32; i < n; i += 32) wts[warp][i] = fast_exp2((ls[(int64_t)i * p.hq] - lse) * kLog2e);
    __syncwarp();
    if (vec) {
        float4 acc[NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < n; i += PF) {  // PF parts x NJ chunks in flight, added in part order
#pragma unroll
            for (int x = 0; x < PF; ++x)
                if (i + x < n) {
                    const float w = wts[warp][i + x];
#pragma unroll
                    for (int j = 0; j < NJ; ++j) fma4(acc[j], w, b[x][j]);
                }
            if (i + PF < n) load(i + PF);
        }
#pragma unroll
        for (int j = 0; j < NJ; ++j)
            if (on[j]) store4<T>(o + c_lo + 128 * j + lane * 4, acc[j]);
    } else {
        for (int c = c_lo + lane; c < c_hi; c += 32) {
            float acc = 0.f;
            for (int i = 0; i < n; ++i) acc += wts[warp][i] * op[i * step + c];
            o[c] = from_f32<T>(acc);
        }
    }
    if (lane == 0 && blockIdx.z == 0) p.lse[row] = lse;
}

template <typename T>
void combine_launch_t(const AttnParams& p, dim3 grid, dim3 block, cudaStream_t st) {
    const int cols = min(p.dv, kCombineCols);  // columns per warp
    if (cols <= 128) combine_kernel<T, 1><<<grid, block, 0, st>>>(p);
    else if (cols <= 256) combine_kernel<T, 2><<<grid, block, 0, st>>>(p);
    else combine_kernel<T, 4><<<grid, block, 0, st>>>(p);
}

cudaError_t launch_combine(const AttnParams& p, pa_dtype dt, cudaStream_t st) {
    if (p.num_cunits == 0) return cudaSuccess;
    const dim3 grid(p.num_cunits, (p.hq + kCombineWarps - 1) / kCombineWarps, (p.dv + kCombineCols - 1) / kCombineCols);
    const dim3 block(kCombineWarps * 32);
    switch (dt) {
        case PA_F32: combine_launch_t<float>(p, grid, block, st); break;
        case PA_BF16: combine_launch_t<__nv_bfloat16>(p, grid, block, st); break;
        default: combine_launch_t<__half>(p, grid, block, st); break;
    }
    return cudaGetLastError();
}

}  // namespace pa
