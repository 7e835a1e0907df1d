// Single translation unit for libbsa.so: the device status word is shared by every
// kernel without relocatable device code.
#include "common.cu"
#include "attention.cu"
#include "routing.cu"
#include "partition.cu"
#include "scoring.cu"
#include "topp.cu"
#include "probe.cu"
#include "repair.cu"
#include "cache.cu"
#include "repair_noalloc.cu"
