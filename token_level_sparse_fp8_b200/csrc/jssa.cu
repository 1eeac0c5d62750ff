// Single translation unit of libjssa.so: the kernels share the device error word defined in
// api.cu, and one unit keeps that a plain (non-relocatable) device symbol.
#include "api.cu"
#include "store.cu"
#include "score_topk.cu"
#include "attend.cu"
#include "gather.cu"
#include "mla.cu"
#include "calib.cu"
#include "basis.cu"
#include "noalloc.cu"
