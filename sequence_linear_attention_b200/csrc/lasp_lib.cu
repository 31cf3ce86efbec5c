// The whole library is one translation unit, so that the per-device status
// word and wait limit (lasp_common.cuh) need no relocatable device code.
#include "lasp_api.cu"
#include "lasp_gla_api.cu"
#include "k_state_scan.cu"
#include "k_simt.cu"
#include "k_tc_states.cu"
#include "k_tc_out.cu"
#include "k_tc_fwd_walk.cu"
#include "k_tc_bwd.cu"
#include "k_tc_bwd_walk.cu"
#include "k_tc_bidir.cu"
#include "k_gla_simt.cu"
#include "lasp_noalloc.cu"
