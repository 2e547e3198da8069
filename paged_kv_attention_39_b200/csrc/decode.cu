// Split-KV paged decode on the tensor cores (bf16 / fp16, head_dim 64, 128 or 256, Dv == D).
//
// A CTA owns one KvUnit for one KV head: up to 16 rows (the queries of a sequence times the
// G query heads that share the KV head) against keys [t0, t1). The K/V bytes of a key are
// read once for the whole GQA group -- no per-head KV repeat, no padded gather: the block
// table is resolved per key row and each 16-byte piece of the row goes straight from its page
// into shared memory with cp.async (zero-filled past t1).
//
// Each warp streams its own tiles of 16*MT keys through a STAGES-deep ring (two stages at D = 64
// and 128, three at D = 256) and keeps its own online-softmax state:
//   S^T[key, row]  = K_tile . Q^T      mma.m16n8k16, keys as M, rows as N (K from smem by
//                                      ldmatrix, Q fragments held in registers)
//   softmax        per row (columns), base-2 units, float32 running max/sum; the max is a
//                  3-step shuffle over the lanes that share a column
//   O^T[d, row]   += V^T_tile . P^T    P^T comes from the S^T accumulators through
//                                      movmatrix.trans; V^T from smem by ldmatrix.trans
// The warps' states are merged in shared memory at the end; the CTA writes the final output
// and lse (one part) or a float32 part for the combine kernel.
//
// Shared memory tiles use a 16-byte-chunk XOR swizzle (chunk ^ (row & 7)) so that ldmatrix
// reads are free of bank conflicts.
#include "device_common.cuh"

namespace pa {

namespace {

constexpr int kWarps = 4;

template <int D, int MT, int STAGES>
struct DecodeCfg {
    static constexpr int TT = 16 * MT;         // keys per warp tile
    static constexpr int CH = D / 8;           // 16-byte chunks per key row
    static constexpr int TILE = TT * D;        // elements of one K (or V) tile
    static constexpr int WARP_ELEMS = STAGES * 2 * TILE;
    static constexpr size_t PIPE_BYTES = (size_t)kWarps * WARP_ELEMS * 2;
    static constexpr size_t EPI_BYTES = (size_t)kWarps * (16 * D + 32) * 4;
    static constexpr size_t SMEM = PIPE_BYTES > EPI_BYTES ? PIPE_BYTES : EPI_BYTES;
};

__device__ __forceinline__ int swz(int row, int chunk) { return chunk ^ (row & 7); }

}  // namespace

// The merge of a split (row set, KV head), run by the CTA whose part completes it last (ruDNN
// "merge FP32 statistics"; alice-llm `lse_combine`): for each of the R rows, lse = logsumexp_i
// lse_i over its parts and out = sum_i exp(lse_i - lse) o_i, parts taken in index order, so the
// result does not depend on which CTA merges. A row whose parts are all empty gets out = 0 and
// lse = -inf. Every CTA publishes its part (fence, then one counted arrival); the CTA that sees
// the count complete reads the parts from L2 and puts the counter back to zero.
template <typename T, int D>
__device__ __forceinline__ void merge_own_parts(const AttnParams& p, const KvUnit& u, const SeqInfo& si, int kvh,
                                                int R) {
    __shared__ int s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float kLog2e = 1.4426950408889634f;
    int* ctr = p.merge_ctr + (int64_t)u.part_base * p.hkv + kvh;
    __threadfence();  // this CTA's part is visible before its arrival is counted
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(ctr, 1) == u.nsplit - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();  // the parts counted before this arrival are visible to this CTA
    const int G = p.group;
    const int64_t step = (int64_t)p.hq * D;
    for (int r = warp; r < R; r += kWarps) {
        const int j = u.j0 + r / G, h = kvh * G + r % G;
        const int64_t base = (int64_t)u.part_base + (int64_t)(j - u.j0) * u.nsplit;
        const float* ls = p.ws_lse + base * p.hq + h;  // part i at ls[i * hq]
        const float* op = p.ws_o + (base * p.hq + h) * D;
        const int64_t qrow = (int64_t)(si.q_start + j) * p.hq + h;
        T* o = static_cast<T*>(p.out) + qrow * D;
        // up to 32 parts: lane i keeps part i's lse and weight, handed out by shuffles; more parts
        // are read again per use
        const int n = u.nsplit;
        const float my_l = lane < n ? __ldcg(ls + (int64_t)lane * p.hq) : neg_inf();
        float m = my_l;
        for (int i = lane + 32; i < n; i += 32) m = fmaxf(m, __ldcg(ls + (int64_t)i * p.hq));
        m = warp_max(m);
        if (m == neg_inf()) {
            for (int d = lane; d < D; d += 32) o[d] = from_f32<T>(0.f);
            if (lane == 0) p.lse[qrow] = m;
            continue;
        }
        float sum = lane < n ? fast_exp2((my_l - m) * kLog2e) : 0.f;
        for (int i = lane + 32; i < n; i += 32) sum += fast_exp2((__ldcg(ls + (int64_t)i * p.hq) - m) * kLog2e);
        sum = warp_sum(sum);
        const float lse = m + __logf(sum);
        const float my_w = lane < n ? fast_exp2((my_l - lse) * kLog2e) : 0.f;
        auto weight = [&](int i) {
            return i < 32 ? __shfl_sync(0xffffffffu, my_w, i)
                          : fast_exp2((__ldcg(ls + (int64_t)i * p.hq) - lse) * kLog2e);
        };
        for (int d0 = 0; d0 < D; d0 += 128) {
            const int d = d0 + lane * 4;
            const bool on = d < D;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            int i = 0;
            for (; i + 4 <= n; i += 4) {  // four parts in flight, added in part order
                float4 b[4];
                float w[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    w[x] = weight(i + x);
                    b[x] = on ? __ldcg(reinterpret_cast<const float4*>(op + (i + x) * step + d))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    acc.x = fmaf(w[x], b[x].x, acc.x);
                    acc.y = fmaf(w[x], b[x].y, acc.y);
                    acc.z = fmaf(w[x], b[x].z, acc.z);
                    acc.w = fmaf(w[x], b[x].w, acc.w);
                }
            }
            for (; i < n; ++i) {
                const float w = weight(i);
                const float4 b = on ? __ldcg(reinterpret_cast<const float4*>(op + i * step + d))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                acc.x = fmaf(w, b.x, acc.x);
                acc.y = fmaf(w, b.y, acc.y);
                acc.z = fmaf(w, b.z, acc.z);
                acc.w = fmaf(w, b.w, acc.w);
            }
            if (on) {
                uint2 v;
                v.x = pack2<T>(acc.x, acc.y);
                v.y = pack2<T>(acc.z, acc.w);
                *reinterpret_cast<uint2*>(o + d) = v;
            }
        }
        if (lane == 0) p.lse[qrow] = lse;
    }
    if (threadIdx.x == 0) *ctr = 0;  // ready for the next call
}

template <typename T, int D, int NT, int MT, int STAGES, bool SPARSE>
__global__ void __launch_bounds__(kWarps * 32) decode_mma_kernel(const AttnParams p) {
    using C = DecodeCfg<D, MT, STAGES>;
    constexpr int TT = C::TT, CH = C::CH, KK = D / 16;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    T* smem = reinterpret_cast<T*>(smem_raw);

    const KvUnit u = p.units[blockIdx.x];
    const int kvh = blockIdx.y;
    const SeqInfo si = p.seqs[u.seq];
    const int G = p.group;
    const int R = (u.j1 - u.j0) * G;  // live rows, <= 8 * NT
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, tq = lane & 3;  // fragment row group / thread-in-group
    // Sparse: one query per unit; its keys are reached through the selection row of (query, kvh)
    // and a tile of TT keys never straddles two blocks (TT divides block_size and t0).
    const int32_t* selrow = nullptr;
    if constexpr (SPARSE) selrow = p.sel + ((int64_t)(si.q_start + u.j0) * p.hkv + kvh) * p.sel_width;
    const int bs = p.block_size;

    // ---- query fragments (B operand of S^T = K Q^T): column n = row gq of the n-tile ------
    uint32_t qf[NT][KK][2];
    const T* qp = static_cast<const T*>(p.q);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int r = nt * 8 + gq;
        const bool live = r < R;
        const int j = u.j0 + (live ? r / G : 0);
        const int64_t qrow = (int64_t)(si.q_start + j) * p.hq + kvh * G + (live ? r % G : 0);
        const uint32_t* src = reinterpret_cast<const uint32_t*>(qp + qrow * D);
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            qf[nt][kk][0] = live ? src[kk * 8 + tq] : 0u;
            qf[nt][kk][1] = live ? src[kk * 8 + 4 + tq] : 0u;
        }
    }
    // absolute positions of this thread's two columns per n-tile (padding rows: visible)
    int64_t posc[NT][2];
    bool livec[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = nt * 8 + 2 * tq + e;
            livec[nt][e] = r < R;
            posc[nt][e] = (int64_t)si.L - si.n + u.j0 + (r < R ? r / G : 0);
        }
    // keys every live row can see: [all_lo, all_hi)
    const int64_t p_min = (int64_t)si.L - si.n + u.j0;
    const int64_t p_max = (int64_t)si.L - si.n + u.j1 - 1;
    const int64_t all_lo = p.window > 0 ? p_max - p.window + 1 : INT64_MIN;
    const int64_t all_hi = p.causal ? p_min + 1 : INT64_MAX;

    float m_run[NT][2], l_run[NT][2];
    float o[KK][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = neg_inf();
        l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
        for (int dt = 0; dt < KK; ++dt) o[dt][nt][0] = o[dt][nt][1] = o[dt][nt][2] = o[dt][nt][3] = 0.f;
    }

    T* wbuf = smem + (size_t)warp * C::WARP_ELEMS;
    const T* kc = static_cast<const T*>(p.k);
    const T* vc = static_cast<const T*>(p.v);
    const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
    const int ps = p.page_size;
    const int64_t rstride = (int64_t)p.hkv * D;
    const int ntiles = (u.t1 - u.t0 + TT - 1) / TT;
    const int my_tiles = ntiles > warp ? (ntiles - warp + kWarps - 1) / kWarps : 0;

    auto load_tile = [&](int it, int stage) {
        const int tok0 = u.t0 + (warp + it * kWarps) * TT;
        int64_t off = -1;
        if (lane < TT) {
            if constexpr (SPARSE) {
                const int vk = tok0 + lane;
                if (vk < u.t1) {
                    const int32_t blk = selrow[vk / bs];
                    const int64_t t = (int64_t)blk * bs + vk % bs;
                    if (blk >= 0 && t < si.L) off = ((int64_t)bt[t / ps] * ps + t % ps) * rstride + (int64_t)kvh * D;
                }
            } else {
                const int t = tok0 + lane;
                if (t < u.t1) off = ((int64_t)bt[t / ps] * ps + t % ps) * rstride + (int64_t)kvh * D;
            }
        }
        T* dk = wbuf + stage * 2 * C::TILE;
        T* dv = dk + C::TILE;
#pragma unroll
        for (int c = lane; c < TT * CH; c += 32) {
            const int row = c / CH, ch = c % CH;
            const int64_t ro = __shfl_sync(0xffffffffu, off, row);
            const bool ok = ro >= 0;
            const int64_t src = ok ? ro + ch * 8 : 0;
            const int dst = row * D + swz(row, ch) * 8;
            cp_async_16(dk + dst, kc + src, ok);
            cp_async_16(dv + dst, vc + src, ok);
        }
    };

#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        if (s < my_tiles) load_tile(s, s);
        cp_async_commit();
    }

    for (int it = 0; it < my_tiles; ++it) {
        {
            const int nx = it + STAGES - 1;
            if (nx < my_tiles) load_tile(nx, nx % STAGES);
            cp_async_commit();
        }
        cp_async_wait<STAGES - 1>();
        __syncwarp();
        const int stage = it % STAGES;
        const T* sk = wbuf + stage * 2 * C::TILE;
        const T* sv = sk + C::TILE;
        const int tok0 = u.t0 + (warp + it * kWarps) * TT;

        // ---- S^T = K Q^T -------------------------------------------------------------------
        float s[MT][NT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) s[mt][nt][0] = s[mt][nt][1] = s[mt][nt][2] = s[mt][nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KK; ++kk) {
                uint32_t a[4];
                const int row = mt * 16 + (lane & 15);
                ldmatrix_x4(a, sk + row * D + swz(row, kk * 2 + (lane >> 4)) * 8);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816<T>(s[mt][nt], a, qf[nt][kk][0], qf[nt][kk][1]);
            }
        }
        // ---- scale, mask, running max ----------------------------------------------------
        bool full;
        int64_t tbase = tok0;  // position of the tile's first key
        bool tvalid = true;
        if constexpr (SPARSE) {
            const int32_t blk = selrow[tok0 / bs];
            tvalid = blk >= 0;
            tbase = (int64_t)blk * bs + tok0 % bs;
            full = tvalid && tok0 + TT <= u.t1 && tbase + TT <= si.L && tbase >= all_lo && tbase + TT - 1 < all_hi;
        } else {
            full = tok0 + TT <= u.t1 && tok0 >= all_lo && tok0 + TT - 1 < all_hi;
        }
        float tmax[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) tmax[nt][0] = tmax[nt][1] = neg_inf();
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float x = s[mt][nt][e] * p.scale_log2;
                    if (!full) {
                        const int o = mt * 16 + gq + 8 * (e >> 1);
                        const int64_t t = tbase + o;
                        const int c = e & 1;
                        const bool vis = tvalid && tok0 + o < u.t1 && (!SPARSE || t < si.L) &&
                                         (!livec[nt][c] || key_visible(t, posc[nt][c], p.causal, p.window));
                        if (!vis) x = neg_inf();
                    }
                    s[mt][nt][e] = x;
                    tmax[nt][e & 1] = fmaxf(tmax[nt][e & 1], x);
                }
        float alpha[NT][2], muse[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float v = tmax[nt][c];
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                const float m_new = fmaxf(m_run[nt][c], v);
                muse[nt][c] = m_new == neg_inf() ? 0.f : m_new;
                alpha[nt][c] = fast_exp2(m_run[nt][c] - muse[nt][c]);
                m_run[nt][c] = m_new;
                l_run[nt][c] *= alpha[nt][c];
            }
        // ---- probabilities -> B fragments of P^T (movmatrix) --------------------------------
        uint32_t pb[MT][NT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float p0 = fast_exp2(s[mt][nt][0] - muse[nt][0]);
                const float p1 = fast_exp2(s[mt][nt][1] - muse[nt][1]);
                const float p2 = fast_exp2(s[mt][nt][2] - muse[nt][0]);
                const float p3 = fast_exp2(s[mt][nt][3] - muse[nt][1]);
                l_run[nt][0] += p0 + p2;
                l_run[nt][1] += p1 + p3;
                pb[mt][nt][0] = movmatrix_trans(pack2<T>(p0, p1));
                pb[mt][nt][1] = movmatrix_trans(pack2<T>(p2, p3));
            }
        // ---- rescale and accumulate O^T += V^T P^T ----------------------------------------
#pragma unroll
        for (int dt = 0; dt < KK; ++dt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                o[dt][nt][0] *= alpha[nt][0];
                o[dt][nt][1] *= alpha[nt][1];
                o[dt][nt][2] *= alpha[nt][0];
                o[dt][nt][3] *= alpha[nt][1];
            }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int dt = 0; dt < KK; ++dt) {
                uint32_t a[4];
                const int i = lane >> 3;
                const int row = mt * 16 + (lane & 7) + 8 * (i >> 1);
                ldmatrix_x4_trans(a, sv + row * D + swz(row, dt * 2 + (i & 1)) * 8);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816<T>(o[dt][nt], a, pb[mt][nt][0], pb[mt][nt][1]);
            }
        __syncwarp();
    }
    cp_async_wait<0>();

    // ---- merge the warps' states ------------------------------------------------------------
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float v = l_run[nt][c];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            l_run[nt][c] = v;
        }
    __syncthreads();  // pipeline buffers are reused below
    float* eo = reinterpret_cast<float*>(smem_raw);            // [kWarps][16][D]
    float* em = eo + kWarps * 16 * D;                          // [kWarps][16]
    float* el = em + kWarps * 16;                              // [kWarps][16]
#pragma unroll
    for (int dt = 0; dt < KK; ++dt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = dt * 16 + gq + 8 * (e >> 1);
                const int r = nt * 8 + 2 * tq + (e & 1);
                eo[(warp * 16 + r) * D + d] = o[dt][nt][e];
            }
    if (gq == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int r = nt * 8 + 2 * tq + c;
                em[warp * 16 + r] = m_run[nt][c];
                el[warp * 16 + r] = l_run[nt][c];
            }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < R * D; idx += kWarps * 32) {
        const int r = idx / D, d = idx % D;
        float M = neg_inf();
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, em[w * 16 + r]);
        float L = 0.f, O = 0.f;
        if (M != neg_inf()) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float f = fast_exp2(em[w * 16 + r] - M);
                L += el[w * 16 + r] * f;
                O += eo[(w * 16 + r) * D + d] * f;
            }
        }
        const bool empty = !(L > 0.f);
        const float val = empty ? 0.f : O / L;
        const float lse = empty ? neg_inf() : (M + __log2f(L)) * kLn2;
        const int j = u.j0 + r / G;
        const int h = kvh * G + r % G;
        const int64_t qrow = (int64_t)(si.q_start + j) * p.hq + h;
        if (u.nsplit == 1) {
            static_cast<T*>(p.out)[qrow * D + d] = from_f32<T>(val);
            if (d == 0) p.lse[qrow] = lse;
        } else {
            const int64_t slot = (int64_t)u.part_base + (int64_t)(j - u.j0) * u.nsplit + u.split;
            p.ws_o[(slot * p.hq + h) * D + d] = val;
            if (d == 0) p.ws_lse[slot * p.hq + h] = lse;
        }
    }
    if constexpr (!SPARSE) {
        if (p.merge_ctr != nullptr && u.nsplit > 1) merge_own_parts<T, D>(p, u, si, kvh, R);
    }
}

namespace {

template <typename T, int D, int NT, bool SPARSE>
cudaError_t launch_cfg(const AttnParams& p, cudaStream_t st) {
    // Two stages per warp at D = 64 and 128: the smaller ring lets more CTAs share an SM, which
    // hides more latency than a deeper ring per warp (measured on the decode batches: 2 stages
    // 1-3 % faster than 3, and 4 or 5 slower). D = 256 and the sparse variant keep three.
    constexpr int MT = 1, STAGES = ((D == 64 || D == 128) && !SPARSE) ? 2 : 3;
    using C = DecodeCfg<D, MT, STAGES>;
    auto kern = decode_mma_kernel<T, D, NT, MT, STAGES, SPARSE>;
    static unsigned long long configured = 0;  // one bit per device ordinal
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    kern<<<dim3(p.num_units, p.hkv), kWarps * 32, C::SMEM, st>>>(p);
    return cudaGetLastError();
}

template <typename T, bool SPARSE>
cudaError_t launch_t(const AttnParams& p, int rows_max, cudaStream_t st) {
    const bool two = rows_max > 8;
    if (p.d == 64) return two ? launch_cfg<T, 64, 2, SPARSE>(p, st) : launch_cfg<T, 64, 1, SPARSE>(p, st);
    if (p.d == 256) return two ? launch_cfg<T, 256, 2, SPARSE>(p, st) : launch_cfg<T, 256, 1, SPARSE>(p, st);
    return two ? launch_cfg<T, 128, 2, SPARSE>(p, st) : launch_cfg<T, 128, 1, SPARSE>(p, st);
}

}  // namespace

cudaError_t launch_decode_mma(const AttnParams& p, pa_dtype dt, int rows_max, cudaStream_t st) {
    if (p.num_units == 0) return cudaSuccess;
    if (p.sel) {
        if (dt == PA_BF16) return launch_t<__nv_bfloat16, true>(p, rows_max, st);
        return launch_t<__half, true>(p, rows_max, st);
    }
    if (dt == PA_BF16) return launch_t<__nv_bfloat16, false>(p, rows_max, st);
    return launch_t<__half, false>(p, rows_max, st);
}

}  // namespace pa
