// abi_util.cuh -- host-side argument checks and the failure-injection hook
// shared by every extern "C" entry point of the library.
#pragma once

#include <cstdlib>
#include <cstring>

#include "common.cuh"

namespace dspark {

inline bool dtype_ok(int dt) { return dt == DSPARK_F32 || dt == DSPARK_BF16; }
inline bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }
// bf16 arrays are read by TMA and 16-byte vector loads.
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Shape and dtype limits of the drafting and verification calls.
inline dspark_status check_common(int B, int G, int V, int r, int dtype) {
    if (!dtype_ok(dtype)) return DSPARK_ERR_UNSUPPORTED_DTYPE;
    if (B < 1 || B > 4096 || G < 1 || G > 16 || V < 2 || V > (1 << 20) || r < 1 || r > 512)
        return DSPARK_ERR_INVALID_ARG;
    // bf16 rows are moved by TMA: 16-byte row pitches for the logits and factors.
    if (dtype == DSPARK_BF16 && ((r % 16) != 0 || (V % 8) != 0)) return DSPARK_ERR_INVALID_ARG;
    return DSPARK_OK;
}

inline dspark_status check_ws(const void *ws, size_t have, size_t need) {
    if (ws == nullptr || !aligned256(ws) || have < need) return DSPARK_ERR_WORKSPACE;
    return DSPARK_OK;
}

// Host-side fault injection for failure-path tests: DSPARK_INJECT_ERROR=<entry
// point name>=<status> makes that entry point return <status> without
// enqueuing work.
inline dspark_status injected(const char *name) {
    const char *env = getenv("DSPARK_INJECT_ERROR");
    if (env == nullptr) return DSPARK_OK;
    const size_t n = strlen(name);
    if (strncmp(env, name, n) == 0 && env[n] == '=') return (dspark_status)atoi(env + n + 1);
    return DSPARK_OK;
}

}  // namespace dspark
