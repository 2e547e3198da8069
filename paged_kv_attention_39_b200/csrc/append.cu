// Paged K/V append (ruDNN `DevicePlan::append`): the new keys/values of every query row are
// written into their page slots before attention runs. Query j of sequence s (n_s queries,
// L_s keys including the new ones) owns absolute position p = L_s - n_s + j, i.e. page
// block_tables[s][p / page_size], slot p % page_size. The rows of all KV heads of one query are
// contiguous both in the new rows ([q][h][:]) and in the slot ([slot][h][:]), so one warp copies
// one query: its K bytes and then its V bytes as one run of 16-byte pieces, eight pieces per lane
// loaded before any is stored. Queries are independent: a pure HBM stream.
#include "device_common.cuh"

namespace pa {

constexpr int kAppendWarps = 8;
constexpr int kAppendUnroll = 8;  // 16-byte pieces in flight per lane

__global__ void __launch_bounds__(kAppendWarps * 32)
    append_kernel(const uint8_t* __restrict__ new_k, const uint8_t* __restrict__ new_v, uint8_t* __restrict__ k_cache,
                  uint8_t* __restrict__ v_cache, const SeqInfo* __restrict__ seqs, const int32_t* __restrict__ q2seq,
                  const int32_t* __restrict__ block_tables, int32_t table_width, int32_t page_size, int32_t hkv,
                  int32_t k_row_bytes, int32_t v_row_bytes, int64_t num_queries) {
    const int64_t qi = (int64_t)blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    if (qi >= num_queries) return;
    const int lane = threadIdx.x & 31;
    const int32_t s = q2seq[qi];
    const SeqInfo si = seqs[s];
    const int64_t pos = (int64_t)si.L - si.n + (qi - si.q_start);
    const int64_t slot = (int64_t)block_tables[(int64_t)s * table_width + pos / page_size] * page_size + pos % page_size;
    const int64_t kq = (int64_t)hkv * k_row_bytes, vq = (int64_t)hkv * v_row_bytes;  // bytes per query
    const uint4* sk = reinterpret_cast<const uint4*>(new_k + qi * kq);
    const uint4* sv = reinterpret_cast<const uint4*>(new_v + qi * vq);
    uint4* dk = reinterpret_cast<uint4*>(k_cache + slot * kq);
    uint4* dv = reinterpret_cast<uint4*>(v_cache + slot * vq);
    const int64_t nk = kq / 16, n = nk + vq / 16;  // pieces: K first, then V
    for (int64_t base = lane; base < n; base += 32 * kAppendUnroll) {
        uint4 t[kAppendUnroll];
#pragma unroll
        for (int u = 0; u < kAppendUnroll; ++u) {
            const int64_t i = base + u * 32;
            if (i < nk) t[u] = sk[i];
            else if (i < n) t[u] = sv[i - nk];
        }
#pragma unroll
        for (int u = 0; u < kAppendUnroll; ++u) {
            const int64_t i = base + u * 32;
            if (i < nk) dk[i] = t[u];
            else if (i < n) dv[i - nk] = t[u];
        }
    }
}

cudaError_t launch_append(const void* new_k, const void* new_v, void* k_cache, void* v_cache, const SeqInfo* seqs,
                          const int32_t* q2seq, const int32_t* block_tables, int32_t table_width, int32_t page_size,
                          int32_t hkv, int32_t k_row_bytes, int32_t v_row_bytes, int64_t rows, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    const int64_t num_queries = rows / hkv;  // rows = queries x KV heads
    const int64_t blocks = (num_queries + kAppendWarps - 1) / kAppendWarps;
    append_kernel<<<(unsigned)blocks, kAppendWarps * 32, 0, st>>>(
        static_cast<const uint8_t*>(new_k), static_cast<const uint8_t*>(new_v), static_cast<uint8_t*>(k_cache),
        static_cast<uint8_t*>(v_cache), seqs, q2seq, block_tables, table_width, page_size, hkv, k_row_bytes, v_row_bytes,
        num_queries);
    return cudaGetLastError();
}

}  // namespace pa
