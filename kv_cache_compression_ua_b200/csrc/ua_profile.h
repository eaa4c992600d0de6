// ua_profile.h -- RAII event bracket used around every kernel launch (see ua_profile.cu).
#pragma once
#include <cuda_runtime.h>

namespace ua {

class ProfileScope {
public:
    ProfileScope(const char* name, cudaStream_t s);
    ~ProfileScope();
    ProfileScope(const ProfileScope&) = delete;
    ProfileScope& operator=(const ProfileScope&) = delete;

private:
    int idx_;
    cudaStream_t stream_;
};

}  // namespace ua

#define UA_PROF_CAT2(a, b) a##b
#define UA_PROF_CAT(a, b) UA_PROF_CAT2(a, b)
#define UA_PROFILE(name, stream) ::ua::ProfileScope UA_PROF_CAT(ua_prof_scope_, __LINE__)(name, stream)
