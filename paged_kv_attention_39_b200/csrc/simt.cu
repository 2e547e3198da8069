// CUDA-core paged attention kernel: every dtype (fp32 / bf16 / fp16), every head size up to
// 1024, GQA and MLA. One warp owns one (query, query head) row of a KvUnit and walks that
// unit's keys one at a time: page lookup through the block table, a lane-strided dot product
// reduced with warp shuffles, an online softmax in base-2 units with float32 statistics and
// accumulators, then either the final output/lse or one float32 split part.
//
// This is the exact-precision path (no 16-bit rounding of probabilities), used for fp32 and
// for shapes the tensor-core kernels do not take. With a sparse selection the unit's keys are
// positions in the concatenation of the row's selected blocks (see AttnParams::sel).
#include "device_common.cuh"

namespace pa {

template <typename T, int PL>
__global__ void __launch_bounds__(128) simt_kernel(const AttnParams p) {
    const KvUnit u = p.units[blockIdx.x];
    const int kvh = blockIdx.y;
    const SeqInfo si = p.seqs[u.seq];
    const int G = p.group;
    const int rows = (u.j1 - u.j0) * G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T* __restrict__ qp = static_cast<const T*>(p.q);
    const T* __restrict__ kp = static_cast<const T*>(p.k);
    const T* __restrict__ vp = static_cast<const T*>(p.v);
    const T* __restrict__ qrp = static_cast<const T*>(p.qr);
    const T* __restrict__ krp = static_cast<const T*>(p.kr);
    const int32_t* __restrict__ bt = p.block_tables + (int64_t)u.seq * p.table_width;
    const int ps = p.page_size;

    for (int r = warp; r < rows; r += blockDim.x >> 5) {
        const int j = u.j0 + r / G;
        const int h = kvh * G + r % G;
        const int64_t qrow = (int64_t)(si.q_start + j) * p.hq + h;
        const int64_t pos = (int64_t)si.L - si.n + j;
        float qv[PL], qr[PL], acc[PL];
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int c = lane + 32 * i;
            qv[i] = c < p.d ? to_f32(qp[qrow * p.d + c]) : 0.f;
            qr[i] = c < p.pr ? to_f32(qrp[qrow * p.pr + c]) : 0.f;
            acc[i] = 0.f;
        }
        float m = neg_inf(), l = 0.f;
        const int32_t* selrow = p.sel ? p.sel + ((int64_t)(si.q_start + j) * p.hkv + kvh) * p.sel_width : nullptr;
        for (int vk = u.t0; vk < u.t1; ++vk) {
            int64_t t = vk;
            if (selrow) {  // sparse: key vk of the concatenated selected blocks
                const int32_t blk = selrow[vk / p.block_size];
                t = (int64_t)blk * p.block_size + vk % p.block_size;
                if (blk < 0 || t >= si.L) {  // nothing left in this block entry
                    vk += p.block_size - 1 - vk % p.block_size;
                    continue;
                }
            }
            if (!key_visible(t, pos, p.causal, p.window)) continue;
            const int64_t slot = (int64_t)bt[t / ps] * ps + t % ps;
            const int64_t krow = (slot * p.hkv + kvh) * p.d;
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int c = lane + 32 * i;
                if (c < p.d) dot += qv[i] * to_f32(kp[krow + c]);
                if (c < p.pr) dot += qr[i] * to_f32(krp[slot * p.pr + c]);
            }
            const float s = warp_sum(dot) * p.scale_log2;
            const float m_new = fmaxf(m, s);
            const float alpha = fast_exp2(m - m_new);
            const float e = fast_exp2(s - m_new);
            l = l * alpha + e;
            const int64_t vrow = (slot * p.hkv + kvh) * p.dv;
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int c = lane + 32 * i;
                const float vv = c < p.dv ? to_f32(vp[vrow + c]) : 0.f;
                acc[i] = acc[i] * alpha + e * vv;
            }
            m = m_new;
        }
        const bool empty = !(l > 0.f);
        const float inv = empty ? 0.f : 1.f / l;
        const float lse = empty ? neg_inf() : (m + __log2f(l)) * kLn2;
        if (u.nsplit == 1) {
            T* o = static_cast<T*>(p.out) + qrow * p.dv;
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int c = lane + 32 * i;
                if (c < p.dv) o[c] = from_f32<T>(acc[i] * inv);
            }
            if (lane == 0) p.lse[qrow] = lse;
        } else {
            const int64_t slot = (int64_t)u.part_base + (int64_t)(j - u.j0) * u.nsplit + u.split;
            float* o = p.ws_o + (slot * p.hq + h) * p.dv;
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int c = lane + 32 * i;
                if (c < p.dv) o[c] = acc[i] * inv;
            }
            if (lane == 0) p.ws_lse[slot * p.hq + h] = lse;
        }
    }
}

template <typename T>
static cudaError_t launch_t(const AttnParams& p, cudaStream_t st) {
    const int widest = max(max(p.d, p.dv), p.pr);
    const dim3 grid(p.num_units, p.hkv), block(128);
    if (widest <= 32) simt_kernel<T, 1><<<grid, block, 0, st>>>(p);
    else if (widest <= 64) simt_kernel<T, 2><<<grid, block, 0, st>>>(p);
    else if (widest <= 128) simt_kernel<T, 4><<<grid, block, 0, st>>>(p);
    else if (widest <= 256) simt_kernel<T, 8><<<grid, block, 0, st>>>(p);
    else if (widest <= 512) simt_kernel<T, 16><<<grid, block, 0, st>>>(p);
    else simt_kernel<T, 32><<<grid, block, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_simt(const AttnParams& p, pa_dtype dt, cudaStream_t st) {
    if (p.num_units == 0) return cudaSuccess;
    switch (dt) {
        case PA_F32: return launch_t<float>(p, st);
        case PA_BF16: return launch_t<__nv_bfloat16>(p, st);
        default: return launch_t<__half>(p, st);
    }
}

}  // namespace pa
