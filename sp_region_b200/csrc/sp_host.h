// Host-side helpers shared by the library's entry points (sp_region.cu,
// sp_gemm.cu): argument validation and the device that owns the data.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "sp_region.h"

namespace spk_host {

struct DevInfo {
    int id;
    int sms;
    int smem_optin;
};

// Make the device that owns `p` current and read its limits.
int use_device_of(const void* p, DevInfo* d);
// The conventions every call shares (sizes, t, dtype, norm, p, eps, rows).
int check_cfg(const sp_cfg* c);
// The token rows [*r0, *r0 + *nrows) a call processes.
void call_rows(const sp_cfg* c, long long* r0, long long* nrows);
int elem_bytes(const sp_cfg* c);
int res_elem_bytes(const sp_cfg* c);
bool aligned(const void* p, size_t a);
// floor(p * 2^32), computed in double
uint32_t drop_threshold(float p);

}  // namespace spk_host
