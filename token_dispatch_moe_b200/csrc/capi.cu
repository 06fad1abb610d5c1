// Library-wide entry points that launch nothing.
#include "common.cuh"

extern "C" const char *moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported size or configuration";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE_INDEX: return "out-of-range id, token or k seen on the device";
        case MOE_ERR_TIMEOUT: return "a bounded device wait timed out";
        case MOE_ERR_NAN_LOGIT: return "NaN logit seen on the device";
    }
    return "unknown status";
}
