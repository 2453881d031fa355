// Single translation unit of libssd.so: the kernels share one module so that
// device-side globals (the status word) are visible to every kernel.
#include "ssd_simt.cu"
#include "ssd_step.cu"
#include "ssd_fused.cu"
#include "ssd_lean.cu"
#include "ssd_pair.cu"
#include "ssd_api.cu"
#include "ssd_noalloc.cu"
#include "ssd_vdecay.cu"
#include "ssd_hostio.cu"
#include "ssd_selftest.cu"
