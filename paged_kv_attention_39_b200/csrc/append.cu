// Paged K/V append (ruDNN `DevicePlan::append`): the new keys/values of every query row are
// written into their page slots before attention runs. Query j of sequence s (n_s queries,
// L_s keys including the new ones) owns absolute position p = L_s - n_s + j, i.e. page
// block_tables[s][p / page_size], slot p % page_size. One warp copies one (query, KV head) row
// of K and V with 16-byte stores; rows are independent, so the kernel is a pure HBM stream.
#include "device_common.cuh"

namespace pa {

constexpr int kAppendWarps = 8;

__global__ void __launch_bounds__(kAppendWarps * 32)
    append_kernel(const uint8_t* __restrict__ new_k, const uint8_t* __restrict__ new_v, uint8_t* __restrict__ k_cache,
                  uint8_t* __restrict__ v_cache, const SeqInfo* __restrict__ seqs, const int32_t* __restrict__ q2seq,
                  const int32_t* __restrict__ block_tables, int32_t table_width, int32_t page_size, int32_t hkv,
                  int32_t k_row_bytes, int32_t v_row_bytes, int64_t rows) {
    const int64_t row = (int64_t)blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31;
    const int64_t qi = row / hkv;
    const int h = (int)(row % hkv);
    const int32_t s = q2seq[qi];
    const SeqInfo si = seqs[s];
    const int64_t pos = (int64_t)si.L - si.n + (qi - si.q_start);
    const int64_t slot = (int64_t)block_tables[(int64_t)s * table_width + pos / page_size] * page_size + pos % page_size;
    const int64_t dst_row = slot * hkv + h;
    const uint4* sk = reinterpret_cast<const uint4*>(new_k + row * k_row_bytes);
    uint4* dk = reinterpret_cast<uint4*>(k_cache + dst_row * k_row_bytes);
    for (int c = lane; c < k_row_bytes / 16; c += 32) dk[c] = sk[c];
    const uint4* sv = reinterpret_cast<const uint4*>(new_v + row * v_row_bytes);
    uint4* dv = reinterpret_cast<uint4*>(v_cache + dst_row * v_row_bytes);
    for (int c = lane; c < v_row_bytes / 16; c += 32) dv[c] = sv[c];
}

cudaError_t launch_append(const void* new_k, const void* new_v, void* k_cache, void* v_cache, const SeqInfo* seqs,
                          const int32_t* q2seq, const int32_t* block_tables, int32_t table_width, int32_t page_size,
                          int32_t hkv, int32_t k_row_bytes, int32_t v_row_bytes, int64_t rows, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    const int64_t blocks = (rows + kAppendWarps - 1) / kAppendWarps;
    append_kernel<<<(unsigned)blocks, kAppendWarps * 32, 0, st>>>(
        static_cast<const uint8_t*>(new_k), static_cast<const uint8_t*>(new_v), static_cast<uint8_t*>(k_cache),
        static_cast<uint8_t*>(v_cache), seqs, q2seq, block_tables, table_width, page_size, hkv, k_row_bytes, v_row_bytes,
        rows);
    return cudaGetLastError();
}

}  // namespace pa
