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
bool make_map_bf16_sw128(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows) {
    return make_map_impl(m, base, rows, cols, box_rows);
}
int sm_count() { return sm_count_impl(); }

}  // namespace xkv
