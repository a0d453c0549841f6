// Host side of the TMA helpers: the driver's tensor-map encoder (looked up once through
// the runtime, so the library needs no link-time dependency on the driver library) and
// the SM count.
#include "sm100_util.cuh"

namespace xkv {
namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)ptr;
    }
    return fn;
}

// 2D bf16 tensor map over a row-major [rows][cols] array with a 128-byte-swizzled box of
// box_rows x 64 elements.
bool make_map_impl(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D view of the same row-major [rows][cols] array: (64 elements, rows, cols / 64
// column blocks) with strides (row: cols * 2 bytes, column block: 128 bytes); a box of
// (64, box_rows, box_cb) lands in shared memory as box_cb consecutive swizzle atoms of
// box_rows x 128 bytes: several 64-column blocks of the same rows in one copy.
bool make_map3_impl(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows, uint32_t box_cb) {
    auto fn = encode_fn();
    if (!fn || cols % 64) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64u, box_rows, box_cb};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count_impl() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

}  // namespace

bool tma_available() { return encode_fn() != nullptr; }
bool make_map_sw128(CUtensorMap *m, const void *base, bool f32, int rank, const uint64_t *dims,
                    const uint64_t *strides, const uint32_t *box) {
    auto fn = encode_fn();
    if (!fn || rank < 1 || rank > 5) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], estr[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        estr[i] = 1;
        if (i + 1 < rank) st[i] = strides[i];
    }
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
              (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool make_map_bf16_sw128(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows) {
    return make_map_impl(m, base, rows, cols, box_rows);
}
bool make_map_bf16_sw128_cb(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                            uint32_t box_rows, uint32_t box_cb) {
    return make_map3_impl(m, base, rows, cols, box_rows, box_cb);
}
int sm_count() { return sm_count_impl(); }

}  // namespace xkv
