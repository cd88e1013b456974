// KDA chunked prefill (placeholder entry points; the kernel follows).
#include "lad_common.cuh"

namespace lad {
int take_device_error_prefill(cudaStream_t, int *code) {
    *code = 0;
    return LAD_OK;
}
}  // namespace lad

extern "C" size_t kda_prefill_workspace_size(int, int, int, int, int, int) { return 0; }

extern "C" int kda_prefill_chunked(const lad_bf16 *, const lad_bf16 *, const lad_bf16 *, const float *, const float *,
                                   float *, void *, int, int, int, int, int, int, float, unsigned, void *, size_t,
                                   void *) {
    return lad::set_error(LAD_EUNSUPPORTED, "kda_prefill_chunked: not built yet");
}
