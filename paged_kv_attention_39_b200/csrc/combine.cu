// Merge of split-KV parts (ruDNN "merge FP32 statistics"; alice-llm `lse_combine`).
// Part i of a row holds its normalised output o_i and logsumexp lse_i over its keys; the
// merged lse is logsumexp_i(lse_i) and the merged output is sum_i exp(lse_i - lse) * o_i.
// Parts without keys carry lse_i = -inf and weight 0; a row whose parts are all empty gets
// out = 0 and lse = -inf. One warp per (query, head); lanes run over the value dimension.
#include "device_common.cuh"

namespace pa {

constexpr int kCombineWarps = 4;
constexpr int kCombineMaxSplits = 1024;

template <typename T>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(const AttnParams p) {
    __shared__ float wts[kCombineWarps][kCombineMaxSplits];
    const CombineUnit cu = p.cunits[blockIdx.x];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y * kCombineWarps + warp;
    if (h >= p.hq) return;
    const int n = cu.nsplit;
    const float* ls = p.ws_lse + (int64_t)cu.part_base * p.hq + h;
    float m = neg_inf();
    for (int i = lane; i < n; i += 32) m = fmaxf(m, ls[(int64_t)i * p.hq]);
    m = warp_max(m);
    const int64_t row = (int64_t)cu.query * p.hq + h;
    T* o = static_cast<T*>(p.out) + row * p.dv;
    if (m == neg_inf()) {
        for (int c = lane; c < p.dv; c += 32) o[c] = from_f32<T>(0.f);
        if (lane == 0) p.lse[row] = m;
        return;
    }
    const float kLog2e = 1.4426950408889634f;
    float sum = 0.f;
    for (int i = lane; i < n; i += 32) sum += fast_exp2((ls[(int64_t)i * p.hq] - m) * kLog2e);
    sum = warp_sum(sum);
    const float lse = m + __logf(sum);
    for (int i = lane; i < n; i += 32) wts[warp][i] = fast_exp2((ls[(int64_t)i * p.hq] - lse) * kLog2e);
    __syncwarp();
    const float* op = p.ws_o + ((int64_t)cu.part_base * p.hq + h) * p.dv;
    const int64_t step = (int64_t)p.hq * p.dv;
    for (int c = lane; c < p.dv; c += 32) {
        float acc = 0.f;
        for (int i = 0; i < n; ++i) acc += wts[warp][i] * op[i * step + c];
        o[c] = from_f32<T>(acc);
    }
    if (lane == 0) p.lse[row] = lse;
}

cudaError_t launch_combine(const AttnParams& p, pa_dtype dt, cudaStream_t st) {
    if (p.num_cunits == 0) return cudaSuccess;
    const dim3 grid(p.num_cunits, (p.hq + kCombineWarps - 1) / kCombineWarps), block(kCombineWarps * 32);
    switch (dt) {
        case PA_F32: combine_kernel<float><<<grid, block, 0, st>>>(p); break;
        case PA_BF16: combine_kernel<__nv_bfloat16><<<grid, block, 0, st>>>(p); break;
        default: combine_kernel<__half><<<grid, block, 0, st>>>(p); break;
    }
    return cudaGetLastError();
}

}  // namespace pa
