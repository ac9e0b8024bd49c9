from . import pipe_peaks, stream_peaks

print(pipe_peaks())
print(stream_peaks())
