// Sparse top-K block selection (alice-llm sparse_attention/llama3_bridge.rs,
// `llama3_sparse_attention`): proxy block scores, top-K selection, and the check/compaction of a
// selection before attention runs over the selected blocks (the attention itself is the split-KV
// decode path reading keys through the selection, followed by the logsumexp merge).
//
// Proxy scores. Block b of sequence s holds keys [b * bs, min((b + 1) * bs, L_s)). For query i
// and KV head h the proxy query is query head h * G; the block's score is the largest
// scale * q_proxy . k_t over the keys t of the block the query sees, -inf if none. The pass is an
// HBM stream of the K rows with float32 dot products of the stored values. 16-bit rows of 64, 128
// or 256 elements (at most 32 KV heads) take the products on the tensor cores (mma.sync, float32
// accumulation), a CTA per (query, block) for every KV head. Otherwise, when a cache slot (the Hkv
// rows of one key) fits one warp at 64 bytes per lane, a CTA scores one (query, block) for every
// KV head and each warp reads whole slots; else one warp scores one (query, KV head, block), four
// lanes sharing a key row, or, for rows that are not a multiple of 64 bytes, one lane per key row.
//
// Top-K. One CTA per (query, KV head) row sorts (score, index) pairs packed into 64-bit keys
// (descending score, then ascending index) with a bitonic sort in shared memory, keeps the first
// k and sorts their indices ascending; rows of at most 256 blocks with k <= 32 take a warp each
// and pick the same k keys by k rounds of a warp minimum.
#include "device_common.cuh"

namespace pa {

namespace {

constexpr int kProxyWarps = 4;
constexpr int kTopkThreads = 256;
constexpr int kPrepThreads = 128;

struct ProxyParams {
    const void* q;
    const void* k;
    float* scores;  // [Nq, Hkv, sw]
    const SeqInfo* seqs;
    const int32_t* q2seq;
    const int32_t* block_tables;
    int32_t table_width, page_size, hq, hkv, group, d, block_size, sw;
    float scale;
    int32_t causal, window;
};

// Keys of block b the query at `pos` sees: [lo, hi) (empty when lo >= hi).
__device__ __forceinline__ void block_visible(const SeqInfo& si, int64_t pos, int b, int bs, int causal,
                                              int window, int64_t* lo, int64_t* hi) {
    int64_t a = (int64_t)b * bs, e = min64((int64_t)(b + 1) * bs, (int64_t)si.L);
    if (window > 0) a = max64(a, pos - window + 1);
    if (causal) e = min64(e, pos + 1);
    *lo = a;
    *hi = e;
}

// -0 and +0 score alike (the selection compares values, not bit patterns).
__device__ __forceinline__ float canonical_zero(float x) { return x == 0.0f ? 0.0f : x; }

template <typename T>
__device__ __forceinline__ void widen16(const uint4& u, float* f) {
    if constexpr (std::is_same<T, float>::value) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    } else {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const unsigned short a = (unsigned short)(w[i] & 0xffffu), b = (unsigned short)(w[i] >> 16);
            if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                f[2 * i] = __bfloat162float(__ushort_as_bfloat16(a));
                f[2 * i + 1] = __bfloat162float(__ushort_as_bfloat16(b));
            } else {
                f[2 * i] = __half2float(__ushort_as_half(a));
                f[2 * i + 1] = __half2float(__ushort_as_half(b));
            }
        }
    }
}

// CPL 16-byte chunks per lane, four lanes per key row (row bytes = 64 * CPL).
template <typename T, int CPL>
__global__ void __launch_bounds__(kProxyWarps * 32) proxy_scores_kernel(const ProxyParams p) {
    constexpr int EPC = 16 / (int)sizeof(T);  // elements per chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const int b = blockIdx.y * kProxyWarps + warp;
    if (b >= p.sw) return;
    const int64_t qi = row / p.hkv;
    const int kvh = (int)(row % p.hkv);
    const int32_t s = p.q2seq[qi];
    const SeqInfo si = p.seqs[s];
    float* out = p.scores + row * p.sw;
    const int nb = (si.L + p.block_size - 1) / p.block_size;
    const int64_t pos = (int64_t)si.L - si.n + (qi - si.q_start);
    int64_t lo = 0, hi = 0;
    if (b < nb) block_visible(si, pos, b, p.block_size, p.causal, p.window, &lo, &hi);
    if (lo >= hi) {
        if (lane == 0) out[b] = neg_inf();
        return;
    }
    const int quarter = lane & 3, kr = lane >> 2;
    float qf[CPL][EPC];
    const T* qp = static_cast<const T*>(p.q) + (qi * p.hq + (int64_t)kvh * p.group) * p.d;
#pragma unroll
    for (int j = 0; j < CPL; ++j) widen16<T>(*reinterpret_cast<const uint4*>(qp + (j * 4 + quarter) * EPC), qf[j]);
    const T* kc = static_cast<const T*>(p.k);
    const int32_t* bt = p.block_tables + (int64_t)s * p.table_width;
    const int ps = p.page_size;
    float m = neg_inf();
#pragma unroll 2
    for (int64_t base = lo; base < hi; base += 8) {  // the same trip count on every lane
        const int64_t t = base + kr;
        const bool live = t < hi;
        float dot = 0.f;
        if (live) {
            const int64_t slot = (int64_t)bt[t / ps] * ps + t % ps;
            const T* kp = kc + (slot * p.hkv + kvh) * p.d;
            uint4 raw[CPL];
#pragma unroll
            for (int j = 0; j < CPL; ++j) raw[j] = __ldg(reinterpret_cast<const uint4*>(kp + (j * 4 + quarter) * EPC));
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                float kf[EPC];
                widen16<T>(raw[j], kf);
#pragma unroll
                for (int e = 0; e < EPC; ++e) dot = fmaf(qf[j][e], kf[e], dot);
            }
        }
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        if (live) m = fmaxf(m, dot);
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    if (lane == 0) out[b] = canonical_zero(m * p.scale);  // scale > 0: the max commutes with it
}

// Any head size: one lane per key row, scalar loads (shapes the chunked kernel does not take).
template <typename T>
__global__ void __launch_bounds__(kProxyWarps * 32) proxy_scores_generic_kernel(const ProxyParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const int b = blockIdx.y * kProxyWarps + warp;
    if (b >= p.sw) return;
    const int64_t qi = row / p.hkv;
    const int kvh = (int)(row % p.hkv);
    const int32_t s = p.q2seq[qi];
    const SeqInfo si = p.seqs[s];
    float* out = p.scores + row * p.sw;
    const int nb = (si.L + p.block_size - 1) / p.block_size;
    const int64_t pos = (int64_t)si.L - si.n + (qi - si.q_start);
    int64_t lo = 0, hi = 0;
    if (b < nb) block_visible(si, pos, b, p.block_size, p.causal, p.window, &lo, &hi);
    const T* qp = static_cast<const T*>(p.q) + (qi * p.hq + (int64_t)kvh * p.group) * p.d;
    const T* kc = static_cast<const T*>(p.k);
    const int32_t* bt = p.block_tables + (int64_t)s * p.table_width;
    float m = neg_inf();
    for (int64_t t = lo + lane; t < hi; t += 32) {
        const int64_t slot = (int64_t)bt[t / p.page_size] * p.page_size + t % p.page_size;
        const T* kp = kc + (slot * p.hkv + kvh) * p.d;
        float dot = 0.f;
        for (int c = 0; c < p.d; ++c) dot = fmaf(to_f32(qp[c]), to_f32(kp[c]), dot);
        m = fmaxf(m, dot);
    }
    m = warp_max(m);
    if (lane == 0) out[b] = m == neg_inf() ? m : canonical_zero(m * p.scale);
}

// Every KV head of one (query, block) in one CTA: a key's cache slot (its Hkv rows, contiguous) is
// read by one warp in one pass, lane l taking 64 bytes of row l / LPR (LPR = row bytes / 64 lanes
// per row), so each load instruction of a warp covers whole 128-byte lines. Warp w takes keys
// lo + w, lo + w + kProxyAllWarps, ..., kProxyUnroll of them per step with all their loads in flight;
// the LPR partial dot products of a row meet by shuffles, and the warps' maxima in shared memory.
// Page arithmetic in 32 bits (positions are below 2^31).
constexpr int kProxyAllWarps = 4;
constexpr int kProxyUnroll = 4;

template <typename T, int LPR>
__global__ void __launch_bounds__(kProxyAllWarps * 32) proxy_scores_slot_kernel(const ProxyParams p) {
    constexpr int EPC = 16 / (int)sizeof(T);  // elements per 16-byte chunk
    constexpr int CPL = 4;                    // chunks per lane: 64 bytes
    __shared__ float wmax[kProxyAllWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t qi = blockIdx.x;  // rows on x (no 65535 limit), blocks on y (at most 16384)
    const int b = blockIdx.y;
    const int32_t s = p.q2seq[qi];
    const SeqInfo si = p.seqs[s];
    const int nb = (si.L + p.block_size - 1) / p.block_size;
    const int64_t pos = (int64_t)si.L - si.n + (qi - si.q_start);
    const int h = lane / LPR, part = lane % LPR;
    const bool head_lane = h < p.hkv;
    float* out = p.scores + qi * p.hkv * (int64_t)p.sw + b;  // + head * sw
    int64_t lo64 = 0, hi64 = 0;
    if (b < nb) block_visible(si, pos, b, p.block_size, p.causal, p.window, &lo64, &hi64);
    if (lo64 >= hi64) {
        if (warp == 0 && part == 0 && head_lane) out[(int64_t)h * p.sw] = neg_inf();
        return;
    }
    const int lo = (int)lo64, hi = (int)hi64;
    float qf[CPL][EPC];
    const T* qp = static_cast<const T*>(p.q) + (qi * p.hq + (int64_t)(head_lane ? h : 0) * p.group) * p.d + part * CPL * EPC;
#pragma unroll
    for (int j = 0; j < CPL; ++j) widen16<T>(*reinterpret_cast<const uint4*>(qp + j * EPC), qf[j]);
    const T* kc = static_cast<const T*>(p.k) + (int64_t)(head_lane ? h : 0) * p.d + part * CPL * EPC;
    const int32_t* bt = p.block_tables + (int64_t)s * p.table_width;
    const int ps = p.page_size;
    const int64_t slot_elems = (int64_t)p.hkv * p.d;
    float m = neg_inf();
    for (int t0 = lo + warp; t0 < hi; t0 += kProxyAllWarps * kProxyUnroll) {
        uint4 raw[kProxyUnroll][CPL];
#pragma unroll
        for (int u = 0; u < kProxyUnroll; ++u) {
            const int t = t0 + u * kProxyAllWarps;
            if (t < hi && head_lane) {
                const int64_t slot = (int64_t)bt[t / ps] * ps + t % ps;
                const T* kp = kc + slot * slot_elems;
#pragma unroll
                for (int j = 0; j < CPL; ++j) raw[u][j] = __ldg(reinterpret_cast<const uint4*>(kp + j * EPC));
            } else {
#pragma unroll
                for (int j = 0; j < CPL; ++j) raw[u][j] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < kProxyUnroll; ++u) {
            float dot = 0.f;
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                float kf[EPC];
                widen16<T>(raw[u][j], kf);
#pragma unroll
                for (int e = 0; e < EPC; ++e) dot = fmaf(qf[j][e], kf[e], dot);
            }
#pragma unroll
            for (int o = 1; o < LPR; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (t0 + u * kProxyAllWarps < hi) m = fmaxf(m, dot);
        }
    }
    wmax[warp][lane] = m;
    __syncthreads();
    if (warp == 0 && part == 0 && head_lane) {
        float mm = wmax[0][lane];
#pragma unroll
        for (int w = 1; w < kProxyAllWarps; ++w) mm = fmaxf(mm, wmax[w][lane]);
        out[(int64_t)h * p.sw] = canonical_zero(mm * p.scale);  // scale > 0: the max commutes with it
    }
}

// (score, index) -> key that sorts ascending as (score descending, index ascending).
__device__ __forceinline__ unsigned long long rank_key(float score, int idx) {
    const uint32_t u = __float_as_uint(canonical_zero(score));
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // monotone in the float value
    return ((unsigned long long)(~ord) << 32) | (uint32_t)idx;
}

__device__ void bitonic_sort(unsigned long long* keys, int n) {  // n a power of two
    for (int size = 2; size <= n; size <<= 1)
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const unsigned long long a = keys[lo], c = keys[hi];
                if ((a > c) == up) {
                    keys[lo] = c;
                    keys[hi] = a;
                }
            }
            __syncthreads();
        }
}

__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float* __restrict__ scores, int32_t sw, int32_t* __restrict__ sel, int32_t width,
                const SeqInfo* __restrict__ seqs, const int32_t* __restrict__ q2seq, int32_t hkv, int32_t bs,
                int32_t topk) {
    extern __shared__ unsigned long long keys[];
    const int64_t row = blockIdx.x;
    const SeqInfo si = seqs[q2seq[row / hkv]];
    const int nb = (si.L + bs - 1) / bs;
    const int k = (topk == 0 || topk >= nb) ? nb : topk;
    int32_t* out = sel + row * width;
    if (k == nb) {  // every block: no ranking needed
        for (int i = threadIdx.x; i < width; i += blockDim.x) out[i] = i < nb ? i : -1;
        return;
    }
    int n = 1;
    while (n < nb) n <<= 1;
    const float* sc = scores + row * sw;
    for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = i < nb ? rank_key(sc[i], i) : ~0ull;
    __syncthreads();
    bitonic_sort(keys, n);
    int m = 1;
    while (m < k) m <<= 1;
    for (int i = threadIdx.x; i < m; i += blockDim.x) keys[i] = i < k ? (keys[i] & 0xffffffffull) : ~0ull;
    __syncthreads();
    bitonic_sort(keys, m);
    for (int i = threadIdx.x; i < width; i += blockDim.x) out[i] = i < k ? (int32_t)keys[i] : -1;
}

// The same selection for rows of at most 256 blocks and k <= 32, a warp per row: each lane holds
// the rank keys of blocks lane, lane + 32, ...; k rounds each take the smallest key of the warp
// (the next block in the order above) and retire it, lane r keeping the r-th pick; the picks are
// then written in ascending block order (a pick's place = the number of smaller picks).
constexpr int kTopkWarpRows = 8;   // rows (warps) per CTA
constexpr int kTopkWarpKeys = 8;   // keys per lane: rows of up to 256 blocks

__global__ void __launch_bounds__(kTopkWarpRows * 32)
    topk_warp_kernel(const float* __restrict__ scores, int32_t sw, int32_t* __restrict__ sel, int32_t width,
                     const SeqInfo* __restrict__ seqs, const int32_t* __restrict__ q2seq, int32_t hkv, int32_t bs,
                     int32_t topk, int64_t rows) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kTopkWarpRows + (threadIdx.x >> 5);
    if (row >= rows) return;
    const SeqInfo si = seqs[q2seq[row / hkv]];
    const int nb = (si.L + bs - 1) / bs;
    const int k = (topk == 0 || topk >= nb) ? nb : topk;
    int32_t* out = sel + row * width;
    if (k == nb) {  // every block: no ranking needed
        for (int i = lane; i < width; i += 32) out[i] = i < nb ? i : -1;
        return;
    }
    const float* sc = scores + row * sw;
    unsigned long long key[kTopkWarpKeys];
#pragma unroll
    for (int j = 0; j < kTopkWarpKeys; ++j) {
        const int i = lane + 32 * j;
        key[j] = i < nb ? rank_key(sc[i], i) : ~0ull;
    }
    int mine = -1;  // lane r: the r-th pick
    for (int r = 0; r < k; ++r) {
        unsigned long long m = key[0];
#pragma unroll
        for (int j = 1; j < kTopkWarpKeys; ++j) m = key[j] < m ? key[j] : m;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, m, o);
            m = other < m ? other : m;
        }
        const int idx = (int)(uint32_t)m;
        if (lane == r) mine = idx;
        const bool owner = lane == (idx & 31);
        const int slot = idx >> 5;
#pragma unroll
        for (int j = 0; j < kTopkWarpKeys; ++j) key[j] = (owner && j == slot) ? ~0ull : key[j];
    }
    int place = 0;
    for (int r = 0; r < k; ++r) place += __shfl_sync(0xffffffffu, mine, r) < mine;
    if (lane < k) out[place] = mine;
    for (int i = k + lane; i < width; i += 32) out[i] = -1;
}

// Caller selection -> checked, compacted selection [Nq, Hkv, wout]: entries in [0, nb_s) that
// are not repeats, in their original order, then -1. A bad entry records code 64 in the error
// word and is dropped. A repeat is found through a bitmap of the row's blocks in shared memory.
__global__ void __launch_bounds__(kPrepThreads)
    sparse_prep_kernel(const int32_t* __restrict__ in, int32_t width, int32_t* __restrict__ outsel, int32_t wout,
                       const SeqInfo* __restrict__ seqs, const int32_t* __restrict__ q2seq, int32_t hkv, int32_t bs,
                       int* err) {
    extern __shared__ uint32_t seen[];
    __shared__ int warp_cnt[kPrepThreads / 32];
    const int64_t row = blockIdx.x;
    const SeqInfo si = seqs[q2seq[row / hkv]];
    const int nb = (si.L + bs - 1) / bs;
    const int words = (nb + 31) / 32;
    for (int i = threadIdx.x; i < words; i += blockDim.x) seen[i] = 0u;
    __syncthreads();
    const int32_t* src = in + row * width;
    int32_t* dst = outsel + row * wout;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int base = 0;
    bool bad = false;
    for (int r0 = 0; r0 < width; r0 += blockDim.x) {
        const int i = r0 + threadIdx.x;
        const int32_t b = i < width ? src[i] : -1;
        bool keep = false;
        if (b != -1) {
            if (b < 0 || b >= nb) {
                bad = true;
            } else {
                const uint32_t bit = 1u << (b & 31);
                keep = (atomicOr(&seen[b >> 5], bit) & bit) == 0u;
                bad |= !keep;
            }
        }
        const uint32_t ballot = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) warp_cnt[warp] = __popc(ballot);
        __syncthreads();
        int before = base;
        for (int w = 0; w < warp; ++w) before += warp_cnt[w];
        int total = 0;
        for (int w = 0; w < kPrepThreads / 32; ++w) total += warp_cnt[w];
        if (keep) {
            const int at = before + __popc(ballot & ((1u << lane) - 1u));
            if (at < wout) dst[at] = b;
        }
        base += total;
        __syncthreads();
    }
    for (int i = base + threadIdx.x; i < wout; i += blockDim.x) dst[i] = -1;
    if (bad && err) atomicCAS(err, 0, 64);
}

// Every KV head of one (query, block) in one CTA, the dot products on the tensor cores (16-bit
// keys, D = 64, 128 or 256, at most kProxyMmaHeads KV heads). The warps take (KV head, 512 / D * 8
// keys) pieces of the block; for every 16 keys a warp issues D / 16 mma.m16n8k16 with the keys as
// M (fragment rows g and g + 8 of lane 4 g + t) and the proxy query copied into all 8 columns of N.
// A dot product does not depend on the order of its terms, so each lane loads the 16-byte chunks
// 4 c + t of its keys' rows and of the query straight from global memory (the four lanes of a key
// cover 64 contiguous bytes per load) and feeds words 0, 1 of chunk c as one k-step and words 2, 3
// as the next, on both operands alike. Keys outside [lo, hi) are not loaded and do not enter the
// max; the warps' maxima meet in shared memory.
constexpr int kProxyMmaHeads = 32;

template <typename T, int D>
__global__ void __launch_bounds__(kProxyAllWarps * 32) proxy_scores_mma_kernel(const ProxyParams p) {
    constexpr int CH = D / 32;   // 16-byte chunks of a row per lane
    constexpr int R = 512 / D;   // fragment rows per lane per piece: 8 R keys (64 registers of keys)
    __shared__ float wmax[kProxyAllWarps][kProxyMmaHeads];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t qi = blockIdx.x;  // rows on x (no 65535 limit), blocks on y (at most 16384)
    const int b = blockIdx.y;
    const int32_t s = p.q2seq[qi];
    const SeqInfo si = p.seqs[s];
    const int nb = (si.L + p.block_size - 1) / p.block_size;
    const int64_t pos = (int64_t)si.L - si.n + (qi - si.q_start);
    float* out = p.scores + qi * p.hkv * (int64_t)p.sw + b;  // + head * sw
    int64_t lo64 = 0, hi64 = 0;
    if (b < nb) block_visible(si, pos, b, p.block_size, p.causal, p.window, &lo64, &hi64);
    if (lo64 >= hi64) {
        for (int h = threadIdx.x; h < p.hkv; h += blockDim.x) out[(int64_t)h * p.sw] = neg_inf();
        return;
    }
    const int lo = (int)lo64, hi = (int)hi64;
    for (int h = lane; h < p.hkv; h += 32) wmax[warp][h] = neg_inf();
    __syncwarp();
    const int pieces = (hi - lo + 8 * R - 1) / (8 * R);
    const T* kc = static_cast<const T*>(p.k) + t * 8;
    const int32_t* bt = p.block_tables + (int64_t)s * p.table_width;
    const int ps = p.page_size;
    const int64_t slot_elems = (int64_t)p.hkv * D;
    for (int it = warp; it < p.hkv * pieces; it += kProxyAllWarps) {
        const int h = it % p.hkv, t0 = lo + (it / p.hkv) * 8 * R;
        const T* qp = static_cast<const T*>(p.q) + (qi * p.hq + (int64_t)h * p.group) * D + t * 8;
        uint4 qf[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) qf[c] = __ldg(reinterpret_cast<const uint4*>(qp + c * 32));
        uint4 kf[R][CH];
        bool vis[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {  // fragment row r: key t0 + 8 r + g
            const int tk = t0 + 8 * r + g;
            vis[r] = tk < hi;
            if (vis[r]) {
                const int64_t slot = (int64_t)bt[tk / ps] * ps + tk % ps;
                const T* kp = kc + slot * slot_elems + (int64_t)h * D;
#pragma unroll
                for (int c = 0; c < CH; ++c) kf[r][c] = __ldg(reinterpret_cast<const uint4*>(kp + c * 32));
            } else {
#pragma unroll
                for (int c = 0; c < CH; ++c) kf[r][c] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        float m = neg_inf();
#pragma unroll
        for (int gr = 0; gr < R / 2; ++gr) {  // 16 keys: rows 2 gr (keys g) and 2 gr + 1 (keys g + 8)
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < CH; ++c) {
                const uint4 ka = kf[2 * gr][c], kb = kf[2 * gr + 1][c];
                const uint32_t a0[4] = {ka.x, kb.x, ka.y, kb.y};
                mma16816<T>(d, a0, qf[c].x, qf[c].y);
                const uint32_t a1[4] = {ka.z, kb.z, ka.w, kb.w};
                mma16816<T>(d, a1, qf[c].z, qf[c].w);
            }
            if (vis[2 * gr]) m = fmaxf(m, d[0]);
            if (vis[2 * gr + 1]) m = fmaxf(m, d[2]);
        }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (lane == 0) wmax[warp][h] = fmaxf(wmax[warp][h], m);
    }
    __syncthreads();
    for (int h = threadIdx.x; h < p.hkv; h += blockDim.x) {
        float mm = wmax[0][h];
#pragma unroll
        for (int w = 1; w < kProxyAllWarps; ++w) mm = fmaxf(mm, wmax[w][h]);
        out[(int64_t)h * p.sw] = canonical_zero(mm * p.scale);  // scale > 0: the max commutes with it
    }
}

template <typename T>
cudaError_t proxy_launch_t(const ProxyParams& p, int64_t rows, cudaStream_t st) {
    const int64_t row_bytes = (int64_t)p.d * (int64_t)sizeof(T);
    if constexpr (sizeof(T) == 2) {  // dot products on the tensor cores
        if ((p.d == 64 || p.d == 128 || p.d == 256) && p.hkv <= kProxyMmaHeads) {
            const dim3 g((unsigned)(rows / p.hkv), (unsigned)p.sw);
            if (p.d == 64) proxy_scores_mma_kernel<T, 64><<<g, kProxyAllWarps * 32, 0, st>>>(p);
            else if (p.d == 128) proxy_scores_mma_kernel<T, 128><<<g, kProxyAllWarps * 32, 0, st>>>(p);
            else proxy_scores_mma_kernel<T, 256><<<g, kProxyAllWarps * 32, 0, st>>>(p);
            return cudaGetLastError();
        }
    }
    // whole cache slots per warp when a slot's rows fit one warp at 64 bytes per lane
    const int lpr = row_bytes % 64 == 0 ? (int)(row_bytes / 64) : 0;
    if ((lpr == 1 || lpr == 2 || lpr == 4 || lpr == 8) && (int64_t)p.hkv * lpr <= 32) {
        const dim3 g((unsigned)(rows / p.hkv), (unsigned)p.sw);
        switch (lpr) {
            case 1: proxy_scores_slot_kernel<T, 1><<<g, kProxyAllWarps * 32, 0, st>>>(p); break;
            case 2: proxy_scores_slot_kernel<T, 2><<<g, kProxyAllWarps * 32, 0, st>>>(p); break;
            case 4: proxy_scores_slot_kernel<T, 4><<<g, kProxyAllWarps * 32, 0, st>>>(p); break;
            default: proxy_scores_slot_kernel<T, 8><<<g, kProxyAllWarps * 32, 0, st>>>(p); break;
        }
        return cudaGetLastError();
    }
    const dim3 grid((unsigned)rows, (unsigned)((p.sw + kProxyWarps - 1) / kProxyWarps));
    const int cpr = row_bytes % 16 == 0 ? (int)(row_bytes / 16) : 0;  // 16-byte chunks per row
    switch (cpr % 4 == 0 ? cpr / 4 : 0) {
        case 1: proxy_scores_kernel<T, 1><<<grid, kProxyWarps * 32, 0, st>>>(p); break;
        case 2: proxy_scores_kernel<T, 2><<<grid, kProxyWarps * 32, 0, st>>>(p); break;
        case 4: proxy_scores_kernel<T, 4><<<grid, kProxyWarps * 32, 0, st>>>(p); break;
        case 8: proxy_scores_kernel<T, 8><<<grid, kProxyWarps * 32, 0, st>>>(p); break;
        default: proxy_scores_generic_kernel<T><<<grid, kProxyWarps * 32, 0, st>>>(p); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_scores(const void* q, const void* k, float* scores, int32_t sw, const SeqInfo* seqs,
                                 const int32_t* q2seq, const int32_t* block_tables, int32_t table_width,
                                 int32_t page_size, int32_t hq, int32_t hkv, int32_t d, int32_t block_size,
                                 float scale, int causal, int32_t window, int64_t num_queries, pa_dtype dt,
                                 cudaStream_t st) {
    if (num_queries == 0 || sw == 0) return cudaSuccess;
    ProxyParams p{q, k, scores, seqs, q2seq, block_tables, table_width, page_size, hq, hkv, hq / hkv, d,
                  block_size, sw, scale, causal, window};
    const int64_t rows = num_queries * hkv;
    switch (dt) {
        case PA_F32: return proxy_launch_t<float>(p, rows, st);
        case PA_BF16: return proxy_launch_t<__nv_bfloat16>(p, rows, st);
        default: return proxy_launch_t<__half>(p, rows, st);
    }
}

cudaError_t launch_sparse_topk(const float* scores, int32_t sw, int32_t* sel, int32_t width, const SeqInfo* seqs,
                               const int32_t* q2seq, int32_t hkv, int32_t block_size, int32_t topk,
                               int32_t nb_max, int64_t num_queries, cudaStream_t st) {
    if (num_queries == 0) return cudaSuccess;
    if (nb_max <= 32 * kTopkWarpKeys && topk <= 32) {
        const int64_t rows = num_queries * hkv;
        topk_warp_kernel<<<(unsigned)((rows + kTopkWarpRows - 1) / kTopkWarpRows), kTopkWarpRows * 32, 0, st>>>(
            scores, sw, sel, width, seqs, q2seq, hkv, block_size, topk, rows);
        return cudaGetLastError();
    }
    int n = 1;
    while (n < nb_max) n <<= 1;
    const size_t smem = (size_t)n * sizeof(unsigned long long);
    if (smem > 48 * 1024) {
        static unsigned long long configured = 0;
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev >= 64 || !(configured >> dev & 1ull)) {
            e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(PA_SPARSE_MAX_BLOCKS * sizeof(unsigned long long)));
            if (e != cudaSuccess) return e;
            if (dev < 64) configured |= 1ull << dev;
        }
    }
    topk_kernel<<<(unsigned)(num_queries * hkv), kTopkThreads, smem, st>>>(scores, sw, sel, width, seqs, q2seq, hkv,
                                                                           block_size, topk);
    return cudaGetLastError();
}

cudaError_t launch_sparse_prep(const int32_t* in, int32_t width, int32_t* out, int32_t wout, const SeqInfo* seqs,
                               const int32_t* q2seq, int32_t hkv, int32_t block_size, int32_t nb_max,
                               int64_t num_queries, int* err, cudaStream_t st) {
    if (num_queries == 0 || wout == 0) return cudaSuccess;
    const size_t smem = (size_t)((nb_max + 31) / 32) * sizeof(uint32_t);
    sparse_prep_kernel<<<(unsigned)(num_queries * hkv), kPrepThreads, smem, st>>>(in, width, out, wout, seqs, q2seq,
                                                                                  hkv, block_size, err);
    return cudaGetLastError();
}

}  // namespace pa
