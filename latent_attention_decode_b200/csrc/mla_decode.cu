// Gated MLA latent decode (placeholder entry points; the kernel follows).
#include "lad_common.cuh"

namespace lad {
int take_device_error_mla(cudaStream_t, int *code) {
    *code = 0;
    return LAD_OK;
}
}  // namespace lad

extern "C" size_t mla_latent_decode_workspace_size(int, int, int, int) { return 0; }

extern "C" int mla_latent_decode(const lad_bf16 *, const lad_bf16 *, long long, const int *, const float *, void *,
                                 float *, int, int, int, int, int, float, unsigned, void *, size_t, void *) {
    return lad::set_error(LAD_EUNSUPPORTED, "mla_latent_decode: not built yet");
}
