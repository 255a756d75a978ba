// Host side of the TMA row loads: tensor-map descriptors for row tensors whose rows are
// equally spaced in memory (a dense [R, H] tensor, or a [T, heads, H] view whose token
// stride is heads x the head stride, such as [T,24,256] with strides (12288, 512, 1)).
// One 2-D tiled load then brings P whole rows into shared memory, where per-row bulk
// copies would need P requests.  A TMA box dimension holds at most 256 elements and the
// shared-memory destination of a tensor load must be 128-byte aligned, so only rows of
// H <= 256 with H a multiple of 64 qualify.
#include "common.cuh"

namespace rmsk {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's encoder, looked up once per process (a function-local static: the lookup is
// thread-safe, and the entry point is the same for every device).
EncodeTiledFn encoder() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return nullptr;
    }();
    return fn;
}

}  // namespace

int64_t uniform_row_stride(const RowsIn& v, int heads) {
    if (heads == 1) return v.st;
    if (v.st == (int64_t)heads * v.sk) return v.sk;
    return -1;
}

bool encode_row_map(CUtensorMap* m, const void* base, int H, int64_t rows, int64_t stride,
                    int box_rows) {
    // A tensor load writes shared memory at 128-byte aligned addresses only: rows of a
    // multiple of 128 bytes (H % 64 == 0) keep every slot's region aligned.
    if (H > 256 || H % 64 || stride <= 0 || stride % 8 || rows <= 0 || box_rows < 1 ||
        box_rows > 256 || (reinterpret_cast<uintptr_t>(base) & 15))
        return false;
    EncodeTiledFn fn = encoder();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)stride * 2};  // bytes, multiple of 16
    const cuuint32_t box[2] = {(cuuint32_t)H, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

void make_row_maps(RowMaps* maps, const RowsIn* views, int n, int heads, int H, int64_t rows,
                   int box_rows) {
    for (int i = 0; i < 3; ++i) maps->use[i] = 0;
    for (int i = 0; i < n; ++i) {
        const int64_t stride = uniform_row_stride(views[i], heads);
        maps->use[i] = encode_row_map(&maps->map[i], views[i].ptr, H, rows, stride, box_rows);
    }
}

}  // namespace rmsk
