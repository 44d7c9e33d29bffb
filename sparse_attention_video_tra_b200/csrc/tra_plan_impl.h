// tra_plan_impl.h -- the host-side plan object behind the opaque tra_plan.
#pragma once
#include <cstddef>

#include "tra_geom.h"

struct tra_plan_s {
    tra::Geom geom;        // parameter block handed to every kernel
    double gamma;
    int Rt;
    unsigned flags;
    size_t mask_bytes;
};
