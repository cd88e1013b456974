// Library-wide C-ABI pieces: error strings, version, device error word.
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <vector>

#include "lad_common.cuh"

namespace lad {

static thread_local char g_last_error[512] = "";

int set_error(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return code;
}

int check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return LAD_OK;
}

int device_sm_count() {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= static_cast<int>(cache.size())) cache.resize(dev + 1, 0);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

void *tensor_map_encoder_raw() {
    static std::once_flag once;
    static void *fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = p;
    });
    return fn;
}

}  // namespace lad

extern "C" const char *lad_last_error(void) { return lad::g_last_error; }

extern "C" int lad_version(void) { return 102; }

extern "C" int lad_device_error(void *stream, int *code) {
    if (!code) return lad::set_error(LAD_EINVAL, "lad_device_error: code is NULL");
    cudaStream_t s = lad::as_stream(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return lad::set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    int c1 = 0, c2 = 0, c3 = 0, c4 = 0;
    int rc = lad::take_device_error_mla(s, &c1);
    if (rc != LAD_OK) return rc;
    rc = lad::take_device_error_prefill(s, &c2);
    if (rc != LAD_OK) return rc;
    rc = lad::take_device_error_cache(s, &c3);
    if (rc != LAD_OK) return rc;
    rc = lad::take_device_error_kda(s, &c4);
    if (rc != LAD_OK) return rc;
    *code = c1 ? c1 : (c2 ? c2 : (c3 ? c3 : c4));
    return LAD_OK;
}
