// Specialized row kernels (filled in below as shapes get dedicated kernels).
#include <cuda_runtime.h>

#include "harp_internal.h"

harp_status launch_apply_fast(harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                              int64_t ld_y, harp_dtype in_dtype, harp_dir dir, void* stream,
                              harp_dtype out_dtype) {
    (void)p; (void)x; (void)y; (void)rows; (void)ld_x; (void)ld_y; (void)in_dtype; (void)dir;
    (void)stream; (void)out_dtype;
    return HARP_ERR_UNSUPPORTED;
}

void fast_state_free(harp_plan_s* p) { (void)p; }
