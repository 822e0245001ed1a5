// Status strings and version of libmoe.
#include "common.cuh"

MOE_API const char *moe_status_str(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null pointer or inconsistent size";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape outside the supported range";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: kernel launch rejected";
        case MOE_ERR_OVERFLOW: return "MOE_ERR_OVERFLOW: size product overflows";
        case MOE_ERR_HOST: return "MOE_ERR_HOST: host memory or a host thread could not be had";
    }
    return "MOE_ERR_UNKNOWN";
}

MOE_API int moe_version(void) { return 100; }
