// Single translation unit of libgdn.so: every kernel and the C ABI.
#include "gdn_status.cu"
#include "gdn_ffma.cu"
#include "gdn_tc.cu"
#include "gdn_ring.cu"
#include "gdn_seq.cu"
#include "gdn_bidir.cu"
#include "gdn_attn.cu"
#include "gdn_api.cu"
