// Single translation unit of libsage2: the kernels share one device error word
// (sage2::g_device_error), which whole-program CUDA compilation only allows
// inside one translation unit.
#include "quant.cu"
#include "corr.cu"
#include "debug_qk.cu"
#include "attn.cu"
#include "api.cu"
#include "noalloc.cu"
#include "varlen.cu"
#include "host_pipe.cu"
