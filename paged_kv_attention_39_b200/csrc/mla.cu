// MLA absorbed-latent paged decode on the 5th-generation tensor cores (bf16 / fp16, latent
// width R = 512, rope width P = 64, up to 128 heads, one query per sequence).
//
// Scores s[h, t] = scale * (q_lat[h] . latent[t] + q_rope[h] . rope[t]) take one M = 128 (heads)
// by N = 32 (keys) by K = R + P = 576 product; the latent rows are also the values, so the same
// shared-memory tile feeds O += P V. The float32 output of 128 heads x 512 columns would fill
// all 512 TMEM columns, leaving none for the scores, so each key range is handled by a pair of
// CTAs: both compute the (identical) scores and softmax, and each accumulates one 256-column
// half of O (TMEM: two score buffers of four 32-column partials + 256 columns of O). The pair's
// second read of a K/V tile comes mostly from L2.
//
//   warp 4      TMA producer: Q (two boxes: 128 heads x all 8 latent column blocks, and the rope
//               part), then per step the latent rows of 32 keys (one box with all 8 column
//               blocks when a page holds the whole step) and the rope rows into a 2-stage ring,
//               with an L2 prefetch a few steps ahead (one box per two steps when a page holds
//               both)
//   warps 5..8  S = Q K^T, nine of the 36 k-steps each into a partial score buffer (warp 5 also
//               owns TMEM)
//   warp 9      O_half += P V_half (2 k-steps); zeroes latent rows past the sequence's last key
//               before P V reads them
//   warps 0..3  softmax, thread = head: S row from TMEM, mask at the range edges, running max
//               and sum in float32, P (16-bit, 64-byte swizzled K-major tile) into shared memory
//
// Every mbarrier wait is bounded (sm100::mbar_wait).
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace pa {

using namespace sm100;

namespace {

constexpr int MR = 512;            // latent width
constexpr int MP = 64;             // rope width
constexpr int MK = MR + MP;        // score contraction length
constexpr int MC = MK / 64;        // 128-byte columns of a Q / K row (8 latent + 1 rope)
constexpr int MBM = 128;           // heads per tile
constexpr int MBN = 32;            // keys per step
constexpr int MST = 2;             // K/V stages
constexpr int MDV = MR / 2;        // output columns per CTA
constexpr int kQkWarps = 4;                   // issuers of S = Q K^T, each a quarter of the k-steps
constexpr int kQkSteps = MK / 16 / kQkWarps;  // 9 k-steps per issuer
constexpr int kQkWarp0 = 5, kPvWarp = kQkWarp0 + kQkWarps;
constexpr int kMlaThreads = (kPvWarp + 1) * 32;
constexpr int kPrefetchTiles = 4;             // L2 prefetch distance of the TMA producer (tiles)
constexpr uint32_t kMlaTmemCols = 512;
constexpr uint64_t kMlaWaitNs = 2000000000ull;

struct MlaSmem {
    static constexpr int Q_COL = MBM * 128;          // one 64-wide column of Q: 16 KB
    static constexpr int KV_COL = MBN * 128;         // one 64-wide column of a K/V tile: 4 KB
    static constexpr int Q = 0;
    static constexpr int KV = Q + MC * Q_COL;        // 144 KB
    static constexpr int P = KV + MST * MC * KV_COL; // + 72 KB
    static constexpr int BAR = P + MBM * 64;         // + 8 KB (128 heads x 32 keys, 16-bit)
    static constexpr int BYTES = BAR + 256;
    static constexpr int ALLOC = BYTES + 1024;
};

enum MBar { M_QFULL = 0, M_FULL = 1, M_EMPTY = M_FULL + MST, M_SFULL = M_EMPTY + MST, M_SFREE = M_SFULL + 2,
            M_PFULL = M_SFREE + 2, M_ODONE = M_PFULL + 2, M_COUNT = M_ODONE + 2 };

// 64-byte swizzle K-major descriptor (rows of 32 16-bit elements, 8-row atoms of 512 bytes).
__device__ __forceinline__ uint64_t sdesc_sw64(uint32_t saddr, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;  // leading byte offset: unused for swizzled K-major
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)4 << 61;  // 64-byte swizzle
    return d;
}

}  // namespace

template <typename T>
__global__ void __launch_bounds__(kMlaThreads, 1)
    mla_tc_kernel(const __grid_constant__ CUtensorMap tm_ql, const __grid_constant__ CUtensorMap tm_qr,
                  const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_latw,
                  const __grid_constant__ CUtensorMap tm_rope, const __grid_constant__ CUtensorMap tm_latw2,
                  const __grid_constant__ CUtensorMap tm_rope2, const AttnParams p) {
    using L_ = MlaSmem;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t IDESC_QK = idesc_f16(MBM, MBN, kBf16, false, false);
    constexpr uint32_t IDESC_PV = idesc_f16(MBM, MDV, kBf16, false, true);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L_::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + M_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Watchdog wd{abort_flag, p.err, kMlaWaitNs};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const KvUnit u = p.units[blockIdx.x >> 1];
    const int hf = blockIdx.x & 1;  // which half of the 512 output columns
    const SeqInfo si = p.seqs[u.seq];
    const int H = p.hq;
    const int64_t qi = si.q_start;          // one query per sequence on this path
    const int64_t pos = (int64_t)si.L - 1;  // its absolute position
    const int ps = p.page_size;
    const int box = ps < MBN ? ps : MBN;
    const int64_t kt_start = ((int64_t)u.t0 / box) * box;
    const int n_tiles = u.t1 > kt_start ? (int)((u.t1 - kt_start + MBN - 1) / MBN) : 0;

    if (tid == 0) {
        for (int i = 0; i < M_COUNT; ++i) {
            uint32_t cnt = 1;
            if (i == M_SFREE || i == M_SFREE + 1 || i == M_PFULL || i == M_PFULL + 1) cnt = 128;
            if (i == M_SFULL || i == M_SFULL + 1) cnt = kQkWarps;
            if (i >= M_EMPTY && i < M_EMPTY + MST) cnt = kQkWarps + 1;
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kQkWarp0) {
        tmem_alloc(tmem_slot, kMlaTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // score buffer b, partial g (one per QK issuer): columns 128 b + 32 g; O: columns 256 .. 511
    const uint32_t t_o = tmem + 256;
    const uint32_t s_base = smem_u32(smem);

    if (warp == 4) {
        // ===================== TMA producer =====================
        // Whole warp in the loop, lane 0 issues; page ids of the next 32 boxes come from one
        // lane-parallel block-table read.
        if (n_tiles > 0) {
            if (lane == 0) {
                tma_prefetch(&tm_ql);
                tma_prefetch(&tm_qr);
                tma_prefetch(&tm_lat);
                tma_prefetch(&tm_latw);
                tma_prefetch(&tm_rope);
                mbar_arrive_expect_tx(&bars[M_QFULL], MC * L_::Q_COL);
                // all 8 latent columns of the 128 heads in one box: [column][head][64 elements]
                tma_load_4d(smem + L_::Q, &tm_ql, &bars[M_QFULL], 0, 0, 0, (int)qi);
                tma_load_3d(smem + L_::Q + (MC - 1) * L_::Q_COL, &tm_qr, &bars[M_QFULL], 0, 0, (int)qi);
            }
            const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
            const int bpt = MBN / box;
            int base_g = -(1 << 30), my_row = 0;
            int issued = 0;
            for (int i = 0; i < n_tiles; ++i) {
                const int64_t kt0 = kt_start + (int64_t)i * MBN;
                int nb = 0;
                for (int b = 0; b < bpt; ++b)
                    if (kt0 + (int64_t)b * box < si.L) nb = b + 1;
                const int g0 = i * bpt;
                if (g0 + (kPrefetchTiles + 1) * bpt > base_g + 32) {  // ids of this tile and the prefetched one
                    base_g = g0;
                    const int64_t key = kt_start + (int64_t)(base_g + lane) * box;
                    my_row = key < si.L ? (int)((int64_t)bt[key / ps] * ps + key % ps) : 0;
                }
                // Warm L2 with the tile kPrefetchTiles ahead: with only two stages, a load issued
                // when a stage frees up would otherwise pay the full HBM latency. Every TMA box
                // costs the copy engine a fixed time, so when a page holds two whole tiles one box
                // of 64 rows prefetches both (issued for the tile that starts the pair).
                const bool pair_pf = bpt == 1 && ps % (2 * box) == 0;
                if (pair_pf) {
                    // one box of two tiles, issued for the tile that starts a page pair
                    const int tp = i + kPrefetchTiles;
                    if (tp < n_tiles && ((kt_start / box + tp) & 1) == 0) {
                        const int prow = __shfl_sync(0xffffffffu, my_row, g0 + kPrefetchTiles - base_g);
                        if (lane == 0) {
                            tma_prefetch_l2_3d(&tm_latw2, 0, prow, 0);
                            tma_prefetch_l2_3d(&tm_rope2, 0, 0, prow);
                        }
                    }
                } else if (i + kPrefetchTiles < n_tiles) {
                    const int gp = g0 + kPrefetchTiles * bpt;
                    const int64_t ktp = kt0 + (int64_t)kPrefetchTiles * MBN;
                    for (int b = 0; b < bpt; ++b) {
                        const int prow = __shfl_sync(0xffffffffu, my_row, gp + b - base_g);
                        if (lane == 0 && ktp + (int64_t)b * box < si.L) {
                            if (bpt == 1) {
                                tma_prefetch_l2_3d(&tm_latw, 0, prow, 0);
                            } else {
                                for (int c = 0; c < MC - 1; ++c) tma_prefetch_l2_3d(&tm_lat, c * 64, 0, prow);
                            }
                            tma_prefetch_l2_3d(&tm_rope, 0, 0, prow);
                        }
                    }
                }
                const int st = i % MST;
                if (i >= MST && !__all_sync(0xffffffffu, mbar_wait(&bars[M_EMPTY + st], ((i / MST) - 1) & 1, wd, 21)))
                    break;
                if (lane == 0) mbar_arrive_expect_tx(&bars[M_FULL + st], (uint32_t)nb * box * 128 * MC);
                uint8_t* dst = smem + L_::KV + st * MC * L_::KV_COL;
                for (int b = 0; b < nb; ++b) {
                    const int row = __shfl_sync(0xffffffffu, my_row, g0 + b - base_g);
                    if (lane == 0) {
                        if (bpt == 1) {  // one page box holds the whole tile: 8 latent columns in one load
                            tma_load_3d(dst, &tm_latw, &bars[M_FULL + st], 0, row, 0);
                        } else {
                            for (int c = 0; c < MC - 1; ++c)
                                tma_load_3d(dst + c * L_::KV_COL + b * box * 128, &tm_lat, &bars[M_FULL + st], c * 64,
                                            0, row);
                        }
                        tma_load_3d(dst + (MC - 1) * L_::KV_COL + b * box * 128, &tm_rope, &bars[M_FULL + st], 0, 0, row);
                    }
                }
                issued = i + 1;
            }
            if (lane == 0 && *abort_flag) {
                const uint64_t t0 = globaltimer_ns();
                auto drain = [&](uint64_t* bar, uint32_t parity) {
                    while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < kMlaWaitNs) {}
                };
                drain(&bars[M_QFULL], 0);
                for (int i = max(0, issued - MST); i < issued; ++i) drain(&bars[M_FULL + i % MST], (i / MST) & 1);
            }
        }
    } else if (warp >= kQkWarp0 && warp < kPvWarp) {
        // ===================== S = Q K^T issuers =====================
        // Each of the kQkWarps warps issues one quarter of the 36 k-steps into its own partial
        // score buffer: a single chain of N = 32 MMAs pays the per-step latency 36 times, four
        // chains from four warps overlap on the tensor core. The softmax adds the partials.
        const int g = warp - kQkWarp0;
        const uint64_t dQ = sdesc_sw128(s_base + L_::Q, 16, 1024);
        const uint64_t dKV = sdesc_sw128(s_base + L_::KV, 16, 1024);
        bool ok = __all_sync(0xffffffffu, n_tiles == 0 || mbar_wait(&bars[M_QFULL], 0, wd, 23));
        for (int i = 0; ok && i < n_tiles; ++i) {
            const int st = i % MST, b = i & 1;
            ok = mbar_wait(&bars[M_FULL + st], (i / MST) & 1, wd, 24);
            if (ok && i >= 2) ok = mbar_wait(&bars[M_SFREE + b], ((i >> 1) - 1) & 1, wd, 25);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t d_s = tmem + b * 128 + g * 32;
                const uint64_t dKst = desc_add(dKV, st * MC * L_::KV_COL);
#pragma unroll
                for (int s2 = 0; s2 < kQkSteps; ++s2) {
                    const int kk = g * kQkSteps + s2;
                    mma_f16_ss(d_s, desc_add(dQ, (kk >> 2) * L_::Q_COL + (kk & 3) * 32),
                               desc_add(dKst, (kk >> 2) * L_::KV_COL + (kk & 3) * 32), IDESC_QK, s2 > 0);
                }
                mma_commit(&bars[M_SFULL + b]);
                mma_commit(&bars[M_EMPTY + st]);
            }
            __syncwarp();
        }
    } else if (warp == kPvWarp) {
        // ===================== O_half += P V_half issuer =====================
        const uint64_t dV = sdesc_sw128(s_base + L_::KV, L_::KV_COL, 1024);
        const uint64_t dP = sdesc_sw64(s_base + L_::P, 512);
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j % MST;
            bool ok = mbar_wait(&bars[M_FULL + st], (j / MST) & 1, wd, 24);
            if (ok) ok = mbar_wait(&bars[M_PFULL + (j & 1)], (j >> 1) & 1, wd, 26);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            // latent rows past the sequence's end hold arbitrary bytes and are values too; the
            // scores of tile j (which read them as keys, masked) are complete by now
            const int64_t kt0 = kt_start + (int64_t)j * MBN;
            const int nvalid = (int)min64(MBN, si.L - kt0);
            if (nvalid < MBN) {
                for (int c = 0; c < MC - 1; ++c) {
                    uint4* col = reinterpret_cast<uint4*>(smem + L_::KV + (st * MC + c) * L_::KV_COL);
                    for (int x = nvalid * 8 + lane; x < MBN * 8; x += 32) col[x] = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            tc_fence_after();
            if (lane == 0) {
                const uint64_t dVs = desc_add(dV, (st * MC + hf * (MDV / 64)) * L_::KV_COL);
                const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < MBN / 16; ++kk)
                    mma_f16_ss(t_o, desc_add(dP, kk * 32), desc_add(dVs, kk * 16 * 128), IDESC_PV, kk > 0 ? 1u : acc0);
                mma_commit(&bars[M_ODONE + (j & 1)]);
                mma_commit(&bars[M_EMPTY + st]);
            }
            __syncwarp();
        }
    } else {
        // ===================== softmax: thread = head =====================
        const int r = tid;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const bool live = r < H;
        const int64_t vis_lo = p.window > 0 ? max64(u.t0, pos - p.window + 1) : u.t0;
        const int64_t vis_hi = p.causal ? min64(u.t1, pos + 1) : u.t1;
        float m_run = neg_inf(), l_run = 0.f;
        bool ok = true;
        for (int i = 0; i < n_tiles; ++i) {
            const int b = i & 1;
            const int64_t kt0 = kt_start + (int64_t)i * MBN;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[M_SFULL + b], (i >> 1) & 1, wd, 28));
            if (!ok) break;
            tc_fence_after();
            uint32_t v[32], w[32];
            const uint32_t t_sb = tmem + b * 128 + lane_off;
            tmem_ld32(t_sb, v);
            tmem_ld32(t_sb + 32, w);
            tmem_ld_wait(v);
            tmem_regs_ready(w);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) + __uint_as_float(w[e]));
#pragma unroll 1
            for (int g = 2; g < kQkWarps; ++g) {
                tmem_ld32(t_sb + g * 32, w);
                tmem_ld_wait(w);
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) + __uint_as_float(w[e]));
            }
            tc_fence_before();
            mbar_arrive(&bars[M_SFREE + b]);
            // keys of this unit the query sees: [vis_lo, vis_hi), the same for every head
            const bool full = kt0 >= vis_lo && kt0 + MBN <= vis_hi;
            const int off_lo = (int)(kt0 - vis_lo), off_hi = (int)(kt0 - vis_hi);
            float m0 = neg_inf(), m1 = neg_inf();
            if (full) {
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    m0 = fmaxf(m0, __uint_as_float(v[e]));
                    m1 = fmaxf(m1, __uint_as_float(v[e + 1]));
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const bool vis = e + off_lo >= 0 && e + off_hi < 0;
                    v[e] = vis ? v[e] : __float_as_uint(neg_inf());
                }
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    m0 = fmaxf(m0, __uint_as_float(v[e]));
                    m1 = fmaxf(m1, __uint_as_float(v[e + 1]));
                }
            }
            const float m_tile = fmaxf(m0, m1) * p.scale_log2;  // scale > 0 commutes with the max
            const float m_new = fmaxf(m_run, m_tile);
            const bool grow = m_new > m_run + 8.0f;
            const bool rescale = grow && i > 0 && m_run != neg_inf();
            // the single P buffer was last read by P V of tile i - 1
            if (i > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[M_ODONE + ((i - 1) & 1)], ((i - 1) >> 1) & 1, wd, 29));
                if (!ok) break;
            }
            if (__any_sync(0xffffffffu, rescale)) {
                tc_fence_after();
                const float alpha = rescale ? fast_exp2(m_run - m_new) : 1.0f;
#pragma unroll 1
                for (int c = 0; c < MDV / 32; ++c) {
                    uint32_t w[32];
                    tmem_ld32(t_o + lane_off + c * 32, w);
                    tmem_ld_wait(w);
#pragma unroll
                    for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * alpha);
                    tmem_st32(t_o + lane_off + c * 32, w);
                }
                tmem_st_wait();
            }
            if (grow) {
                l_run *= fast_exp2(m_run - m_new);
                m_run = m_new;
            }
            const float nm = -(m_run == neg_inf() ? 0.f : m_run);
            uint32_t pk[16];
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) {  // masked scores are -inf: exp2 gives 0
                const float a0 = fast_exp2(fmaf(__uint_as_float(v[2 * e]), p.scale_log2, nm));
                const float a1 = fast_exp2(fmaf(__uint_as_float(v[2 * e + 1]), p.scale_log2, nm));
                s0 += a0;
                s1 += a1;
                pk[e] = pack2<T>(a0, a1);
            }
            l_run += s0 + s1;
            uint8_t* prow = smem + L_::P + r * 64;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(prow + ((c ^ ((r >> 1) & 3)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[M_PFULL + b]);
        }
        // ---- epilogue ----
        if (ok && n_tiles > 0)
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars[M_ODONE + ((n_tiles - 1) & 1)], ((n_tiles - 1) >> 1) & 1, wd, 30));
        tc_fence_after();
        const bool has = l_run > 0.f;
        const float inv = has ? 1.0f / l_run : 0.f;
        const float lse = has ? (m_run + __log2f(l_run)) * kLn2 : neg_inf();
        const int64_t qrow = qi * H + (live ? r : 0);
        const bool split = u.nsplit > 1;
        const int64_t slot = split ? (int64_t)u.part_base + u.split : 0;
#pragma unroll 1
        for (int c = 0; c < MDV / 32; ++c) {
            uint32_t w[32];
            if (ok && n_tiles > 0) {
                tmem_ld32(t_o + lane_off + c * 32, w);
                tmem_ld_wait(w);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) w[e] = 0u;
            }
            if (!(live && ok)) continue;
            const int col0 = hf * MDV + c * 32;
            if (split) {
                float4* dst = reinterpret_cast<float4*>(p.ws_o + (slot * H + r) * MR + col0);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(__uint_as_float(w[4 * e]) * inv, __uint_as_float(w[4 * e + 1]) * inv,
                                         __uint_as_float(w[4 * e + 2]) * inv, __uint_as_float(w[4 * e + 3]) * inv);
            } else {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack2<T>(__uint_as_float(w[2 * e]) * inv, __uint_as_float(w[2 * e + 1]) * inv);
                uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(p.out) + qrow * MR + col0);
#pragma unroll
                for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
        }
        if (live && ok && hf == 0) {
            if (split) p.ws_lse[slot * H + r] = lse;
            else p.lse[qrow] = lse;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kQkWarp0) {
        tc_fence_after();
        tmem_dealloc(tmem, kMlaTmemCols);
    }
}

// ---------------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 mla_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// Tiled map of 16-bit elements with 128B swizzle: `rank` dims (innermost first), byte strides of
// dims 1.., and the box.
bool mla_encode(CUtensorMap* m, bool bf16, const void* base, int rank, const cuuint64_t* dims,
                const cuuint64_t* strides, const cuuint32_t* boxd) {
    auto fn = mla_encode_fn();
    if (!fn) return false;
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank,
              const_cast<void*>(base), dims, strides, boxd, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over a row-major [d2][d1][d0] tensor of 16-bit elements, box {64, b1, b2}, 128B swizzle.
bool mla_map(CUtensorMap* m, bool bf16, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b1,
             uint32_t b2) {
    auto fn = mla_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t boxd[3] = {64, b1, b2};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base),
              dims, strides, boxd, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
cudaError_t mla_launch_t(const AttnParams& p, cudaStream_t st) {
    const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
    const int ps = p.page_size;
    const int box = ps < MBN ? ps : MBN;
    const uint64_t rows = (uint64_t)p.num_pages * ps;
    CUtensorMap tql, tqr, tlat, tlatw, trope, tlatw2, trope2;
    // Absorbed Q [Nq][H][R] seen as {64 elements, head, 64-column block, query}: one box brings the
    // 8 column blocks of 128 heads, laid out [block][head][64 elements] as the MMA reads them.
    const cuuint64_t qdims[4] = {64, (cuuint64_t)p.hq, MR / 64, (cuuint64_t)p.num_queries};
    const cuuint64_t qstr[3] = {MR * 2, 128, (cuuint64_t)p.hq * MR * 2};
    const cuuint32_t qbox[4] = {64, MBM, MR / 64, 1};
    // Latent cache rows [rows][R] seen as {64 elements, row, 64-column block}: one box brings a page
    // box of keys with all 8 column blocks, laid out [block][key][64 elements].
    const cuuint64_t ldims[3] = {64, rows, MR / 64};
    const cuuint64_t lstr[2] = {MR * 2, 128};
    const cuuint32_t lbox[3] = {64, (cuuint32_t)box, MR / 64};
    const cuuint32_t lbox2[3] = {64, (cuuint32_t)(2 * box), MR / 64};
    if (!mla_encode(&tql, bf16, p.q, 4, qdims, qstr, qbox) ||
        !mla_map(&tqr, bf16, p.qr, MP, p.hq, (uint64_t)p.num_queries, MBM, 1) ||
        !mla_map(&tlat, bf16, p.k, MR, 1, rows, 1, box) || !mla_encode(&tlatw, bf16, p.k, 3, ldims, lstr, lbox) ||
        !mla_map(&trope, bf16, p.kr, MP, 1, rows, 1, box) || !mla_encode(&tlatw2, bf16, p.k, 3, ldims, lstr, lbox2) ||
        !mla_map(&trope2, bf16, p.kr, MP, 1, rows, 1, 2 * box))
        return cudaErrorInvalidValue;
    auto kern = mla_tc_kernel<T>;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, MlaSmem::ALLOC);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    kern<<<2 * p.num_units, kMlaThreads, MlaSmem::ALLOC, st>>>(tql, tqr, tlat, tlatw, trope, tlatw2, trope2, p);
    return cudaGetLastError();
}

}  // namespace

bool mla_tc_supported(pa_dtype dt, int heads, int latent_dim, int rope_dim, int page_size) {
    if (dt == PA_F32 || latent_dim != MR || rope_dim != MP || heads < 1 || heads > MBM) return false;
    if (page_size % 16 != 0) return false;
    if (page_size < MBN ? (MBN % page_size != 0) : (page_size % MBN != 0)) return false;
    return true;
}

cudaError_t launch_mla_tc(const AttnParams& p, pa_dtype dt, cudaStream_t st) {
    if (p.num_units == 0) return cudaSuccess;
    if (dt == PA_BF16) return mla_launch_t<__nv_bfloat16>(p, st);
    return mla_launch_t<__half>(p, st);
}

}  // namespace pa
