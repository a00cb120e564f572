// api.cu -- library-wide entry points: version, error strings, device status.
#include "common.cuh"

#include <string>
#include <mutex>

namespace nvfp4 {

static thread_local std::string g_last_error;

nvfp4_status set_error(nvfp4_status st, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

nvfp4_status check_launch(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(NVFP4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return NVFP4_OK;
}

int num_sms()
{
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

bool make_tmap_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t inner, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace nvfp4

extern "C" int nvfp4_version(void) { return 100; }

extern "C" const char *nvfp4_last_error_string(void) { return nvfp4::g_last_error.c_str(); }

extern "C" int nvfp4_num_sms(void) { return nvfp4::num_sms(); }

extern "C" nvfp4_status nvfp4_read_status(const int32_t *dev_status, int32_t *status_out, void *stream)
{
    NVFP4_REQUIRE(dev_status && status_out, NVFP4_ERR_INVALID_ARG, "nvfp4_read_status: null pointer");
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(status_out, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return nvfp4::check_launch("nvfp4_read_status");
    if (cudaStreamSynchronize(st) != cudaSuccess) return nvfp4::check_launch("nvfp4_read_status");
    return NVFP4_OK;
}
