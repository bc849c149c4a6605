// fa_status.h -- status codes shared by the host and device code of libfa
// (the fa_status enum of include/fa.h; the build puts include/ on the path).
#pragma once
#include "fa.h"
