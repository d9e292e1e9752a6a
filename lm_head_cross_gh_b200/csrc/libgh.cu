// Single translation unit of libgh.so: the kernels share one device status
// word, so the sources are compiled together rather than device-linked.
#include "ce.cu"
#include "ce_ring.cu"
#include "ce_vjp.cu"
#include "linear_ce.cu"
#include "api.cu"
#include "noalloc.cu"
