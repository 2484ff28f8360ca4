"""PT-DiT block attention (GIIM + TCM) on B200: ctypes binding over libptdit.so."""
