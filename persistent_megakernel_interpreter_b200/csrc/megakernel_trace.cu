// The megakernel with per-job timestamps (mk_schedule_opts.trace): the same
// source compiled with MK_TRACE=1 into namespace mk::traced.
#define MK_TRACE 1
#include "megakernel.cu"
