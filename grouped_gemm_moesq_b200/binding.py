def load():
    raise RuntimeError("libmoesq.so not built yet")
