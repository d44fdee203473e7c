// compress.cuh -- multi-head SVD compression of the visual K / V cache.
#pragma once

#include "common.cuh"

namespace kvpack {
namespace compress {

inline kvpack_status prepare_device() { return KVPACK_OK; }

inline size_t workspace_bytes(int units, int T) { (void)units; (void)T; return 256; }

inline kvpack_status run(int units, int T, const uint16_t *X, uint16_t *C_lo, uint16_t *C_hi, uint16_t *B,
                         float *sigma, void *ws, int sms, cudaStream_t st) {
    (void)units; (void)T; (void)X; (void)C_lo; (void)C_hi; (void)B; (void)sigma; (void)ws; (void)sms; (void)st;
    return KVPACK_ERR_UNSUPPORTED;
}

}  // namespace compress
}  // namespace kvpack
