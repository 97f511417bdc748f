// Host-side TMA tensor-map encoding. The driver function is fetched through
// the runtime's entry-point query, so the library needs no link-time
// dependency on libcuda.
#include <mutex>

#include "sm100.cuh"

namespace fdl {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    if (rank < 2 || rank > 5 || ((uintptr_t)base & 15u) || box[0] * 2 != 128)
        return cudaErrorInvalidValue;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (box[i] < 1 || box[i] > 256) return cudaErrorInvalidValue;
    }
    for (int i = 0; i < rank - 1; ++i) {
        s[i] = strides_bytes[i];
        if (s[i] % 16) return cudaErrorInvalidValue;
    }
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                    const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t box_rows, uint32_t box_cols) {
    const uint64_t dims[2] = {cols, rows};
    const uint64_t strides[1] = {cols * 2};
    const uint32_t box[2] = {box_cols, box_rows};
    return make_tmap_bf16(map, base, 2, dims, strides, box);
}

cudaError_t make_tmap_bf16_rows(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                uint32_t box_rows, uint32_t n_chunks) {
    if (cols % 64 || n_chunks < 1 || n_chunks * 64 > cols) return cudaErrorInvalidValue;
    // (element within a 64-wide chunk, row, chunk): one copy lands as n_chunks
    // consecutive [box_rows][64] sub-tiles
    const uint64_t dims[3] = {64, rows, cols / 64};
    const uint64_t strides[2] = {cols * 2, 128};
    const uint32_t box[3] = {64, box_rows, n_chunks};
    return make_tmap_bf16(map, base, 3, dims, strides, box);
}

}  // namespace fdl
