// pa_mla.cuh -- MLA (shared-latent) partition pass.  Placeholder until the
// tcgen05 kernel lands: the MLA entry points report PA_ERR_UNSUPPORTED.
#pragma once

#include "pa_device.cuh"

namespace {
inline int pa_mla_default_parts() { return -1; }
}  // namespace

extern "C" {
size_t pa_mla_workspace_size(const pa_mla_desc *) { return 0; }
pa_status pa_decode_mla(const pa_mla_desc *, const void *, const void *, const int32_t *,
                        const int32_t *, float, void *, void *, size_t, void *) {
  return PA_ERR_UNSUPPORTED;
}
pa_status pa_decode_mla_partition(const pa_mla_desc *, const void *, const void *,
                                  const int32_t *, const int32_t *, float, void *, void *,
                                  size_t, void *) {
  return PA_ERR_UNSUPPORTED;
}
pa_status pa_decode_mla_merge(const pa_mla_desc *, const void *, const void *, const int32_t *,
                              const int32_t *, float, void *, void *, size_t, void *) {
  return PA_ERR_UNSUPPORTED;
}
}
