// Backward of MLA absorbed-latent attention on the 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16 / fp16, latent 512, rope 64 (ruDNN `mla_backward`, recompute-based). MLA is
// single-head attention with the key [latent | rope] (576 columns) and the value latent (512): the
// GQA backward with every query head in one group. With P recomputed from the forward's lse and
// dS' = scale * P (dP - Drow):
//     dP = dO . latent_t,   Drow = dO . out
//     d_latent_t += sum_rows dS' q_latent + P dO   (the latent is both key and value)
//     d_rope_t   += sum_rows dS' q_rope
//     d_q_latent = sum_t dS' latent_t,   d_q_rope = sum_t dS' rope_t
// A sequence's rows (its queries x the heads) form one block of at most 128 rows.
//
// mla_bwd_key_kernel: a CTA pair per 128-key tile, CTA c owning latent columns [256 c, 256 c + 256)
// (CTA 0 also the rope), both computing the tile's scores:
//   S^T  = [lat | rope] [q_lat | q_rope]^T  (M = 128 keys, N = 128 rows, K = 576 in nine 64-column
//                                            chunks streamed through a ring) -> TMEM [0, 128)
//   dP^T = lat dO^T                          (K = 512, the same latent chunks) -> TMEM [128, 256)
//   P^T and dS'^T by the compute warps (thread = key), 16-bit, packed over the first 64 columns of
//   their buffers; CTA 0 also writes dS' to a scratch [row][key] for the dQ kernel
//   d_lat[:, own columns] += P^T dO + dS'^T q_lat  (A from TMEM, B = 64-column chunks of dO and
//                                                   q_lat streamed again, MN-major) -> TMEM [256, 512)
//   d_rope += dS'^T q_rope (CTA 0)                                          -> TMEM [64, 128)
// and adds its finished rows once into the float32 caches with TMA reduce-adds (the only writer of
// those rows: plans whose sequences share pages take the CUDA-core kernel).
// mla_bwd_dq_kernel: a CTA per (sequence, 64-column chunk of [latent | rope]):
//   dQ[:, chunk] = dS' [lat | rope][:, chunk]  (M = 128 rows, N = 64, K = the sequence's keys, 64 per
//                                               step: dS' tiles from the scratch, the chunk's page
//                                               boxes), accumulated in TMEM, written once.
//
// Every wait on an mbarrier is bounded (Watchdog): a stalled pipeline sets the plan's error word and
// the CTA leaves through its normal exit, freeing TMEM.
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace pa {

using namespace sm100;

namespace {

constexpr int MB_KT = kMlaBwdKeyTile;  // keys per key-tile CTA
constexpr int MB_R = 512, MB_P = 64;   // latent, rope widths
constexpr int MB_NS = (MB_R + MB_P) / 64;  // 64-column chunks of the score contraction (8 latent + rope)
constexpr int MB_ST = 4;               // ring stages
constexpr int MB_CHUNK = 128 * 128;    // 128 rows of 64 16-bit columns (128-byte rows)
constexpr int kMbLoadWarp = 4, kMbMmaWarp = 5, kMbThreads = 6 * 32;
constexpr uint64_t kMbWaitNs = 2000000000ull;
constexpr float kMbLog2e = 1.4426950408889634f;

struct MbCfg {
    static constexpr int STAGE = 3 * MB_CHUNK;  // key chunk, q chunk, dO chunk
    static constexpr int RING = 0;
    static constexpr int ROWS = RING + MB_ST * STAGE;  // lse2, drow, lo, hi (128 each) + 2 ints
    static constexpr int ROWS_BYTES = 4 * 128 * 4 + 16;
    static constexpr int BAR = ROWS + ROWS_BYTES;
    static constexpr int BYTES = BAR + 256;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr int T_ST = 0, T_DPT = 128, T_ROPE = 64, T_ACC = 256;
    static constexpr int B_FULL = 0, B_EMPTY = B_FULL + MB_ST, B_ROWS = B_EMPTY + MB_ST, B_SFULL = B_ROWS + 1,
                         B_PFULL = B_SFULL + 1, B_DONE = B_PFULL + 1, B_COUNT = B_DONE + 1;
};
static_assert(MbCfg::ALLOC <= 232448, "shared memory of one CTA");
static_assert((128 * 256 + 128 * 64) * 4 <= MB_ST * MbCfg::STAGE, "the finished rows are staged over the ring");

// dQ kernel: ring of (dS' tile: 128 rows x 64 keys, key tile: 64 keys x 64 columns)
constexpr int MQ_ST = 4;
constexpr int MQ_KB = 64;  // keys per step
struct MqCfg {
    static constexpr int A = MB_CHUNK;          // 16 KB
    static constexpr int B = MQ_KB * 128;       // 8 KB
    static constexpr int STAGE = A + B;
    static constexpr int BAR = MQ_ST * STAGE;
    static constexpr int BYTES = BAR + 256;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr int B_FULL = 0, B_EMPTY = B_FULL + MQ_ST, B_DONE = B_EMPTY + MQ_ST, B_COUNT = B_DONE + 1;
};

__device__ __forceinline__ int mb_swz(int row, int chunk) { return chunk ^ (row & 7); }

template <typename T>
__device__ __forceinline__ T from_bits16(uint32_t b);
template <>
__device__ __forceinline__ __nv_bfloat16 from_bits16<__nv_bfloat16>(uint32_t b) {
    return __ushort_as_bfloat16((unsigned short)b);
}
template <>
__device__ __forceinline__ __half from_bits16<__half>(uint32_t b) {
    return __ushort_as_half((unsigned short)b);
}

}  // namespace

template <typename T>
__global__ void __launch_bounds__(kMbThreads, 1)
    mla_bwd_key_kernel(const __grid_constant__ CUtensorMap tm_ql, const __grid_constant__ CUtensorMap tm_qr,
                       const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_lat,
                       const __grid_constant__ CUtensorMap tm_rope, const __grid_constant__ CUtensorMap tm_dlat,
                       const __grid_constant__ CUtensorMap tm_drope, const MlaBwdTcParams p) {
    using C = MbCfg;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t IDESC_S = idesc_f16(128, 128, kBf16, false, false);
    constexpr uint32_t IDESC_G = idesc_f16(128, 64, kBf16, false, true);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Watchdog wd{abort_flag, p.err, kMbWaitNs};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const MlaKeyTile u = p.tiles[blockIdx.x];
    const int half = blockIdx.y;  // latent columns [256 half, 256 half + 256); half 0 also the rope
    const SeqInfo si = p.seqs[u.seq];
    const int H = p.h;
    const int R = si.n * H;  // the sequence's rows, <= 128
    const int64_t row0 = (int64_t)si.q_start * H;
    const int64_t k0 = u.k0, kmax = min64(k0 + MB_KT, si.L);
    const int64_t base_pos = (int64_t)si.L - si.n;
    const int nprod = half == 0 ? 5 : 4;  // product chunks: four latent (and the rope)
    const int nload = MB_NS + nprod;

    if (tid == 0) {
        for (int i = 0; i < C::B_COUNT; ++i) mbar_init(&bars[i], i == C::B_PFULL ? 128u : 1u);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kMbMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t s_base = smem_u32(smem);
    const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
    const int ps = p.page_size;

    if (warp == kMbLoadWarp) {
        // ===================== loads =====================
        // the rows' statistics first (lanes over the 128 rows; rows past the sequence's see no key)
        float* lse2 = reinterpret_cast<float*>(smem + C::ROWS);
        float* drow = lse2 + 128;
        int* lo = reinterpret_cast<int*>(drow + 128);
        int* hi = lo + 128;
        int lo_max = 0, hi_min = INT32_MAX;
        for (int r = lane; r < 128; r += 32) {
            const bool live = r < R;
            const float l = live ? p.lse[row0 + r] : neg_inf();
            const bool has = live && l != neg_inf();
            const int64_t pos = base_pos + (live ? r / H : 0);
            const int64_t a = p.window > 0 ? max64(0, pos - p.window + 1) : 0;
            const int64_t b = p.causal ? min64(si.L, pos + 1) : si.L;
            lse2[r] = has ? l * kMbLog2e : 0.f;
            drow[r] = has ? p.drow[row0 + r] : 0.f;
            lo[r] = has ? (int)a : 0;
            hi[r] = has ? (int)b : 0;
            lo_max = max(lo_max, lo[r]);
            hi_min = min(hi_min, hi[r]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo_max = max(lo_max, __shfl_xor_sync(0xffffffffu, lo_max, o));
            hi_min = min(hi_min, __shfl_xor_sync(0xffffffffu, hi_min, o));
        }
        if (lane == 0) {
            hi[128] = lo_max;  // every row sees [lo_max, hi_min)
            hi[129] = hi_min;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[C::B_ROWS]);
        // the tile's key rows come one TMA box per page (lane b keeps the cache row of box b)
        const int kbox = ps < MB_KT ? ps : MB_KT;
        const int nbox = (int)((kmax - k0 + kbox - 1) / kbox);
        int my_row = 0;
        if (lane < nbox) {
            const int64_t key = k0 + (int64_t)lane * kbox;
            my_row = bt[key / ps] * ps + (int)(key % ps);
        }
        bool ok = true;
        for (int g = 0; ok && g < nload; ++g) {
            const int st = g % MB_ST;
            if (g >= MB_ST)
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_EMPTY + st], ((g / MB_ST) - 1) & 1, wd, 41));
            if (!ok) break;
            uint8_t* ks = smem + C::RING + st * C::STAGE;
            uint8_t* qs = ks + MB_CHUNK;
            uint8_t* os = qs + MB_CHUNK;
            if (g < MB_NS) {  // score chunk g: keys, q and dO columns [64 g, 64 g + 64) (g = 8: the rope)
                const bool rope = g == MB_NS - 1;
                if (lane == 0)
                    mbar_arrive_expect_tx(&bars[C::B_FULL + st],
                                          (uint32_t)(nbox * kbox * 128 + MB_CHUNK + (rope ? 0 : MB_CHUNK)));
                for (int b = 0; b < nbox; ++b) {
                    const int row = __shfl_sync(0xffffffffu, my_row, b);
                    if (lane == 0)
                        tma_load_3d(ks + b * kbox * 128, rope ? &tm_rope : &tm_lat, &bars[C::B_FULL + st],
                                    rope ? 0 : g * 64, 0, row);
                }
                if (lane == 0) {
                    tma_load_3d(qs, rope ? &tm_qr : &tm_ql, &bars[C::B_FULL + st], rope ? 0 : g * 64, 0, (int)row0);
                    if (!rope) tma_load_3d(os, &tm_do, &bars[C::B_FULL + st], g * 64, 0, (int)row0);
                }
            } else {  // product chunk m: q (and dO) columns of this CTA's latent half, or the rope
                const int m = g - MB_NS;
                const bool rope = m == 4;
                const int col = (half * 4 + m) * 64;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars[C::B_FULL + st], rope ? MB_CHUNK : 2 * MB_CHUNK);
                    tma_load_3d(qs, rope ? &tm_qr : &tm_ql, &bars[C::B_FULL + st], rope ? 0 : col, 0, (int)row0);
                    if (!rope) tma_load_3d(os, &tm_do, &bars[C::B_FULL + st], col, 0, (int)row0);
                }
            }
            __syncwarp();
        }
        if (lane == 0 && *abort_flag) {
            // leave no copy in flight into this CTA's shared memory (bounded, ignoring the flag)
            const uint64_t t0 = globaltimer_ns();
            for (int g = max(0, nload - MB_ST); g < nload; ++g)
                while (!mbar_try_wait(&bars[C::B_FULL + g % MB_ST], (g / MB_ST) & 1) &&
                       globaltimer_ns() - t0 < kMbWaitNs) {}
        }
    } else if (warp == kMbMmaWarp) {
        // ===================== MMA issuer =====================
        bool ok = true;
        for (int g = 0; ok && g < MB_NS; ++g) {
            const int st = g % MB_ST;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_FULL + st], (g / MB_ST) & 1, wd, 42));
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t ks = s_base + C::RING + st * C::STAGE;
                const uint64_t dK = sdesc_sw128(ks, 16, 1024);
                const uint64_t dQ = sdesc_sw128(ks + MB_CHUNK, 16, 1024);
                const uint64_t dO = sdesc_sw128(ks + 2 * MB_CHUNK, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t acc = (g > 0 || kk > 0) ? 1u : 0u;
                    mma_f16_ss(tmem + C::T_ST, desc_add(dK, kk * 32), desc_add(dQ, kk * 32), IDESC_S, acc);
                    if (g < MB_NS - 1)
                        mma_f16_ss(tmem + C::T_DPT, desc_add(dK, kk * 32), desc_add(dO, kk * 32), IDESC_S, acc);
                }
                mma_commit(&bars[C::B_EMPTY + st]);
                if (g == MB_NS - 1) mma_commit(&bars[C::B_SFULL]);
            }
            __syncwarp();
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_PFULL], 0, wd, 43));
        if (ok) tc_fence_after();
        // packed P^T / dS'^T: 16 rows = 8 TMEM columns; B = 64-column chunks, the rows as the contraction
        for (int m = 0; ok && m < nprod; ++m) {
            const int g = MB_NS + m, st = g % MB_ST;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_FULL + st], (g / MB_ST) & 1, wd, 44));
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t qs = s_base + C::RING + st * C::STAGE + MB_CHUNK;
                const uint64_t dQn = sdesc_sw128(qs, MB_CHUNK, 1024);
                const uint64_t dOn = sdesc_sw128(qs + MB_CHUNK, MB_CHUNK, 1024);
                if (m < 4) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        mma_f16_ts(tmem + C::T_ACC + m * 64, tmem + C::T_ST + kk * 8, desc_add(dOn, kk * 16 * 128),
                                   IDESC_G, kk > 0 ? 1u : 0u);
                        mma_f16_ts(tmem + C::T_ACC + m * 64, tmem + C::T_DPT + kk * 8, desc_add(dQn, kk * 16 * 128),
                                   IDESC_G, 1u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_f16_ts(tmem + C::T_ROPE, tmem + C::T_DPT + kk * 8, desc_add(dQn, kk * 16 * 128), IDESC_G,
                                   kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars[C::B_EMPTY + st]);
                if (m == nprod - 1) mma_commit(&bars[C::B_DONE]);
            }
            __syncwarp();
        }
    } else {
        // ===================== compute: thread = key =====================
        const int r0 = warp * 32;
        const uint32_t lane_off = (uint32_t)r0 << 16;
        const int64_t t = k0 + r0 + lane;
        const int64_t tw0 = k0 + r0, tw1 = k0 + r0 + 31;
        const float* lse2 = reinterpret_cast<const float*>(smem + C::ROWS);
        const float* drow = lse2 + 128;
        const int* lo = reinterpret_cast<const int*>(drow + 128);
        const int* hi = lo + 128;
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_ROWS], 0, wd, 45));
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_SFULL], 0, wd, 46)) && ok;
        tc_fence_after();
        const bool full = __all_sync(0xffffffffu, tw1 < kmax && tw0 >= hi[128] && tw1 < hi[129]);
        T* ds = static_cast<T*>(p.ds) + u.koff + r0 + lane;  // this key's scratch column
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {  // rows 32 c .. 32 c + 31
            uint32_t sv[32], dv[32];
            tmem_ld32(tmem + lane_off + C::T_ST + c * 32, sv);
            tmem_ld32(tmem + lane_off + C::T_DPT + c * 32, dv);
            tmem_ld_wait(sv);
            tmem_regs_ready(dv);
            uint32_t pk[16], dk[16];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c * 32 + 4 * q);
                const float4 d4 = *reinterpret_cast<const float4*>(drow + c * 32 + 4 * q);
                const int4 a4 = *reinterpret_cast<const int4*>(lo + c * 32 + 4 * q);
                const int4 b4 = *reinterpret_cast<const int4*>(hi + c * 32 + 4 * q);
                const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dr[4] = {d4.x, d4.y, d4.z, d4.w};
                const int la[4] = {a4.x, a4.y, a4.z, a4.w}, lb[4] = {b4.x, b4.y, b4.z, b4.w};
                float pr[4], dsv[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const bool vis = full || (t >= la[x] && t < lb[x]);
                    const float pv = fast_exp2(fmaf(__uint_as_float(sv[4 * q + x]), p.scale_log2, -lv[x]));
                    pr[x] = vis ? pv : 0.f;
                    dsv[x] = vis ? p.scale * pv * (__uint_as_float(dv[4 * q + x]) - dr[x]) : 0.f;
                }
                pk[2 * q] = pack2<T>(pr[0], pr[1]);
                pk[2 * q + 1] = pack2<T>(pr[2], pr[3]);
                dk[2 * q] = pack2<T>(dsv[0], dsv[1]);
                dk[2 * q + 1] = pack2<T>(dsv[2], dsv[3]);
            }
            // 32 rows -> 16 TMEM columns over columns already read (rows 32 c .. at column 16 c)
            tmem_st16(tmem + lane_off + C::T_ST + c * 16, pk);
            tmem_st16(tmem + lane_off + C::T_DPT + c * 16, dk);
            if (half == 0) {  // the dQ kernel's scratch: dS' of this key for rows 32 c .. 32 c + 31
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = c * 32 + 2 * j;
                    ds[(int64_t)r * p.ds_cols] = from_bits16<T>(dk[j] & 0xffffu);
                    ds[(int64_t)(r + 1) * p.ds_cols] = from_bits16<T>(dk[j] >> 16);
                }
            }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[C::B_PFULL]);

        // ---- epilogue: the tile's finished latent (and rope) rows ----
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_DONE], 0, wd, 47));
        tc_fence_after();
        if (ok) {
            // staged over the ring (every load and product is done): 32-column blocks of the 128 key
            // rows, float32, 128-byte swizzled; blocks 0..7 the latent half, 8..9 the rope
            constexpr int CB = 128 * 128;
            uint8_t* stg = smem + C::RING;
            const int r = r0 + lane;
            const int nblk = half == 0 ? 10 : 8;
#pragma unroll 1
            for (int cb = 0; cb < nblk; ++cb) {
                uint32_t a[32];
                tmem_ld32(tmem + lane_off + (cb < 8 ? C::T_ACC + cb * 32 : C::T_ROPE + (cb - 8) * 32), a);
                tmem_ld_wait(a);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<float4*>(stg + cb * CB + r * 128 + (mb_swz(r, ch) << 4)) =
                        make_float4(__uint_as_float(a[4 * ch]), __uint_as_float(a[4 * ch + 1]),
                                    __uint_as_float(a[4 * ch + 2]), __uint_as_float(a[4 * ch + 3]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int rbox = ps < 32 ? ps : 32;
                for (int b0 = 0; b0 < 32; b0 += rbox) {  // this warp's 32 key rows, one box per page
                    const int64_t key = k0 + r0 + b0;
                    if (key >= kmax) break;
                    const int row = bt[key / ps] * ps + (int)(key % ps);
                    for (int cb = 0; cb < nblk; ++cb) {
                        if (cb < 8)
                            tma_reduce_add_3d(&tm_dlat, stg + cb * CB + (r0 + b0) * 128, half * 256 + cb * 32, 0, row);
                        else
                            tma_reduce_add_3d(&tm_drope, stg + cb * CB + (r0 + b0) * 128, (cb - 8) * 32, 0, row);
                    }
                }
                bulk_commit_group();
                bulk_wait_all();
            }
            __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMbMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <typename T>
__global__ void __launch_bounds__(kMbThreads, 1)
    mla_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_ds, const __grid_constant__ CUtensorMap tm_lat,
                      const __grid_constant__ CUtensorMap tm_rope, const MlaBwdTcParams p) {
    using C = MqCfg;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t IDESC = idesc_f16(128, 64, kBf16, false, true);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Watchdog wd{abort_flag, p.err, kMbWaitNs};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const MlaDqUnit u = p.dq_units[blockIdx.x];
    const int ch = blockIdx.y;  // columns [64 ch, 64 ch + 64) of [latent | rope]
    const bool rope = ch == MB_NS - 1;
    const SeqInfo si = p.seqs[u.seq];
    const int R = si.n * p.h;
    const int64_t row0 = (int64_t)si.q_start * p.h;
    const int nsteps = (u.k1 - u.k0) / MQ_KB;
    const int ps = p.page_size, qbox = ps < MQ_KB ? ps : MQ_KB;
    // key rows of step j the boxes bring: those of pages holding a key of the sequence; the rest, and
    // rows past the sequence's end, are zeroed (dS' is zero there, but 0 * garbage is not)
    auto live_rows = [&](int j) {
        const int64_t t0 = (int64_t)u.k0 + (int64_t)j * MQ_KB;
        return (int)max64(0, min64(MQ_KB, (int64_t)si.L - t0));
    };

    if (tid == 0) {
        for (int i = 0; i < C::B_COUNT; ++i) mbar_init(&bars[i], 1u);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kMbMmaWarp) {
        tmem_alloc(tmem_slot, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t s_base = smem_u32(smem);

    if (warp == kMbLoadWarp) {
        const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
        const int bps = MQ_KB / qbox;
        int base_g = -(1 << 30), my_row = 0;
        bool ok = true;
        for (int j = 0; ok && j < nsteps; ++j) {
            const int st = j % MQ_ST;
            const int64_t t0 = (int64_t)u.k0 + (int64_t)j * MQ_KB;
            const int nb = (live_rows(j) + qbox - 1) / qbox;  // boxes holding a key of the sequence
            const int g0 = j * bps;
            if (g0 + nb > base_g + 32) {
                base_g = g0;
                const int64_t key = u.k0 + (int64_t)(base_g + lane) * qbox;
                my_row = key < si.L ? bt[key / ps] * ps + (int)(key % ps) : 0;
            }
            if (j >= MQ_ST)
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_EMPTY + st], ((j / MQ_ST) - 1) & 1, wd, 51));
            if (!ok) break;
            uint8_t* as = smem + st * C::STAGE;
            uint8_t* bs = as + C::A;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[C::B_FULL + st], (uint32_t)(C::A + nb * qbox * 128));
                tma_load_3d(as, &tm_ds, &bars[C::B_FULL + st], u.koff + j * MQ_KB, 0, 0);
            }
            for (int b = 0; b < nb; ++b) {
                const int row = __shfl_sync(0xffffffffu, my_row, g0 + b - base_g);
                if (lane == 0)
                    tma_load_3d(bs + b * qbox * 128, rope ? &tm_rope : &tm_lat, &bars[C::B_FULL + st],
                                rope ? 0 : ch * 64, 0, row);
            }
            (void)t0;
            __syncwarp();
        }
        if (lane == 0 && *abort_flag) {
            const uint64_t t0 = globaltimer_ns();
            for (int j = max(0, nsteps - MQ_ST); j < nsteps; ++j)
                while (!mbar_try_wait(&bars[C::B_FULL + j % MQ_ST], (j / MQ_ST) & 1) &&
                       globaltimer_ns() - t0 < kMbWaitNs) {}
        }
    } else if (warp == kMbMmaWarp) {
        bool ok = true;
        for (int j = 0; ok && j < nsteps; ++j) {
            const int st = j % MQ_ST;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[C::B_FULL + st], (j / MQ_ST) & 1, wd, 52));
            if (!ok) break;
            tc_fence_after();
            const int nz = live_rows(j);
            if (nz < MQ_KB) {
                uint4* base = reinterpret_cast<uint4*>(smem + st * C::STAGE + C::A);
                for (int c = nz * 8 + lane; c < MQ_KB * 8; c += 32) base[c] = make_uint4(0u, 0u, 0u, 0u);
                fence_proxy_async_smem();
                __syncwarp();
            }
            if (lane == 0) {
                const uint32_t as = s_base + st * C::STAGE;
                const uint64_t dA = sdesc_sw128(as, 16, 1024);            // dS': rows x 64 keys, K-major
                const uint64_t dB = sdesc_sw128(as + C::A, C::B, 1024);   // keys x 64 columns, MN-major
#pragma unroll
                for (int kk = 0; kk < MQ_KB / 16; ++kk)
                    mma_f16_ss(tmem, desc_add(dA, kk * 32), desc_add(dB, kk * 16 * 128), IDESC,
                               (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bars[C::B_EMPTY + st]);
                if (j == nsteps - 1) mma_commit(&bars[C::B_DONE]);
            }
            __syncwarp();
        }
    } else {
        // ===================== epilogue: thread = row =====================
        const int r = warp * 32 + lane;
        bool ok = nsteps == 0 || __all_sync(0xffffffffu, mbar_wait(&bars[C::B_DONE], 0, wd, 53));
        tc_fence_after();
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            if (ok && nsteps > 0) {
                tmem_ld32(tmem + lane_off + c * 32, v);
                tmem_ld_wait(v);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = 0u;
            }
            if (r < R && ok) {
                float* dst = rope ? p.dqr + (row0 + r) * MB_P + c * 32 : p.dql + (row0 + r) * MB_R + ch * 64 + c * 32;
                float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                        __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMbMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

namespace {

template <typename T>
cudaError_t launch_mb(const MlaBwdTcParams& p, int num_tiles, int num_dq_units, int64_t num_queries,
                      cudaStream_t st) {
    const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
    const int ps = p.page_size;
    const uint64_t cache_rows = (uint64_t)p.num_pages * ps;
    const uint64_t rows = (uint64_t)num_queries * p.h;
    const uint32_t kbox = ps < MB_KT ? ps : MB_KT, qbox = ps < MQ_KB ? ps : MQ_KB, rbox = ps < 32 ? ps : 32;
    CUtensorMap tql, tqr, tdo, tlat, trope, tdlat, tdrope, tds, tlat_q, trope_q;
    if (!make_map(&tql, bf16, p.ql, MB_R, 1, rows, 1, 128) || !make_map(&tqr, bf16, p.qr, MB_P, 1, rows, 1, 128) ||
        !make_map(&tdo, bf16, p.dout, MB_R, 1, rows, 1, 128) ||
        !make_map(&tlat, bf16, p.lat, MB_R, 1, cache_rows, 1, kbox) ||
        !make_map(&trope, bf16, p.rope, MB_P, 1, cache_rows, 1, kbox) ||
        !make_map_f32(&tdlat, p.dlat, MB_R, 1, cache_rows, 1, rbox) ||
        !make_map_f32(&tdrope, p.drope, MB_P, 1, cache_rows, 1, rbox) ||
        !make_map(&tds, bf16, p.ds, (uint64_t)p.ds_cols, 128, 1, 128, 1) ||
        !make_map(&tlat_q, bf16, p.lat, MB_R, 1, cache_rows, 1, qbox) ||
        !make_map(&trope_q, bf16, p.rope, MB_P, 1, cache_rows, 1, qbox))
        return cudaErrorInvalidValue;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        e = cudaFuncSetAttribute(mla_bwd_key_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, MbCfg::ALLOC);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(mla_bwd_dq_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, MqCfg::ALLOC);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    if (num_tiles > 0)
        mla_bwd_key_kernel<T><<<dim3(num_tiles, 2), kMbThreads, MbCfg::ALLOC, st>>>(tql, tqr, tdo, tlat, trope, tdlat,
                                                                                    tdrope, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (num_dq_units > 0)
        mla_bwd_dq_kernel<T><<<dim3(num_dq_units, MB_NS), kMbThreads, MqCfg::ALLOC, st>>>(tds, tlat_q, trope_q, p);
    return cudaGetLastError();
}

}  // namespace

bool mla_backward_tc_supported(pa_dtype dt, int latent_dim, int rope_dim, int num_heads) {
    return (dt == PA_BF16 || dt == PA_F16) && latent_dim == MB_R && rope_dim == MB_P && num_heads >= 1 &&
           num_heads <= 128;
}

cudaError_t launch_mla_backward_tc(const MlaBwdTcParams& p, pa_dtype dt, int num_tiles, int num_dq_units,
                                   int64_t num_queries, cudaStream_t st) {
    if (dt == PA_BF16) return launch_mb<__nv_bfloat16>(p, num_tiles, num_dq_units, num_queries, st);
    return launch_mb<__half>(p, num_tiles, num_dq_units, num_queries, st);
}

}  // namespace pa
