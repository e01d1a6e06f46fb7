// mk_kernel_traced.cu - the step kernel instances with tracing compiled in
// (per-task records and per-region cycle counts), used only while a trace
// buffer is set with mk_set_trace.  Same source as mk_kernel.cu.
#define MK_TRACE 1
#include "mk_kernel.cu"
